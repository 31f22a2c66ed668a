// Attention preparation: the heaviest-first work list and the reordered,
// zero-padded Q/K/V tiles.
//
// Work list: items (b, h, i) sorted by their number of key blocks, largest
// first -- the single-GPU counterpart of the pages' runtime load balancing
// (FVAttn review, section 3.2: the heavy heads set the critical path), which
// here balances the persistent kernel's CTAs instead of ranks.  Counting sort
// in three launches: histogram, descending bucket offsets, scatter.  The order
// among items with the same count is unspecified (it does not change results).
//
// Permutation: Xp[b, h, n', :] = X[b, perm[n'], h, :] for n' < N and zero for
// the padding rows N <= n' < nb*block (FVAttn review, section 3.1: Hilbert
// curve block reordering), so every key/value block is one dense
// [block, d] tile the attention kernel can fetch with a single TMA box.
#include <cuda_bf16.h>

#include "bsa_internal.cuh"

namespace bsa {
namespace {

__global__ void k_hist(const int32_t* __restrict__ row_ptr, int64_t rows, int nb,
                       int32_t* __restrict__ hist, int32_t* err) {
    const int64_t r = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (r >= rows) return;
    int n = row_ptr[r + 1] - row_ptr[r];
    if (n < 0 || n > nb) {                       // malformed mask: record, clamp
        record_error(err, BSA_EDEVICE, (int)r);
        n = n < 0 ? 0 : nb;
    }
    atomicAdd(&hist[n], 1);
}

// bins[n] = number of items with a count greater than n (start of bucket n in
// descending order).  One CTA; nb + 1 buckets.
__global__ void k_bins(const int32_t* __restrict__ hist, int nb, int32_t* __restrict__ bins) {
    __shared__ int wsum[32];
    const int tid = threadIdx.x;
    const int buckets = nb + 1;
    const int per = (buckets + blockDim.x - 1) / blockDim.x;
    // walk buckets from the top: position u corresponds to bucket nb - u
    const int lo = tid * per, hi = min(buckets, lo + per);
    int run = 0;
    for (int u = lo; u < hi; ++u) run += hist[nb - u];
    int incl = run;
    const int lane = tid % 32, wid = tid / 32;
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) wsum[wid] = incl;
    __syncthreads();
    int off = incl - run;
    for (int w = 0; w < wid; ++w) off += wsum[w];
    for (int u = lo; u < hi; ++u) {
        bins[nb - u] = off;
        off += hist[nb - u];
    }
}

__global__ void k_scatter(const int32_t* __restrict__ row_ptr, int64_t rows, int nb,
                          int32_t* __restrict__ bins, int32_t* __restrict__ work) {
    const int64_t r = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (r >= rows) return;
    int n = row_ptr[r + 1] - row_ptr[r];
    n = n < 0 ? 0 : (n > nb ? nb : n);
    const int pos = atomicAdd(&bins[n], 1);
    work[pos] = (int32_t)r;
}

// One thread moves 16 bytes.  Destination rows are visited in (b, n', h)
// order so that consecutive threads read one token's contiguous H*d row.
__global__ void k_permute(const uint4* __restrict__ q, const uint4* __restrict__ k,
                          const uint4* __restrict__ v, uint4* __restrict__ qp, uint4* __restrict__ kp,
                          uint4* __restrict__ vp, const int32_t* __restrict__ perm, int N, int H,
                          int vec_per_row, int64_t npad, int64_t total) {
    const uint4* src = blockIdx.y == 0 ? q : (blockIdx.y == 1 ? k : v);
    uint4* dst = blockIdx.y == 0 ? qp : (blockIdx.y == 1 ? kp : vp);
    for (int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g < total;
         g += (int64_t)gridDim.x * blockDim.x) {
        const int c = (int)(g % vec_per_row);
        int64_t rest = g / vec_per_row;
        const int h = (int)(rest % H);
        rest /= H;
        const int64_t n = rest % npad;
        const int64_t b = rest / npad;
        uint4 val = make_uint4(0u, 0u, 0u, 0u);
        if (n < N) val = __ldg(src + ((b * N + perm[n]) * H + h) * vec_per_row + c);
        dst[((b * H + h) * npad + n) * vec_per_row + c] = val;
    }
}

}  // namespace

cudaError_t launch_worklist(const bsa_plan& p, const int32_t* row_ptr, int32_t* hist, int32_t* bins,
                            int32_t* work, cudaStream_t s) {
    cudaError_t e = cudaMemsetAsync(hist, 0, (size_t)(p.nb + 1) * sizeof(int32_t), s);
    if (e != cudaSuccess) return e;
    const int t = 256;
    const unsigned g = (unsigned)((p.rows + t - 1) / t);
    k_hist<<<g, t, 0, s>>>(row_ptr, p.rows, (int)p.nb, hist, p.d_err);
    k_bins<<<1, 1024, 0, s>>>(hist, (int)p.nb, bins);
    k_scatter<<<g, t, 0, s>>>(row_ptr, p.rows, (int)p.nb, bins, work);
    return cudaGetLastError();
}

cudaError_t launch_permute(const bsa_plan& p, const void* q, const void* k, const void* v, void* qp,
                           void* kp, void* vp, cudaStream_t s, int n_tensors) {
    const int vec_per_row = p.d * 2 / 16;
    const int64_t npad = p.nb * p.block;
    const int64_t total = (int64_t)p.B * npad * p.H * vec_per_row;
    const int t = 256;
    int64_t blocks = (total + t - 1) / t;
    const int64_t cap = (int64_t)p.num_sms * 16;
    if (blocks > cap) blocks = cap;
    dim3 grid((unsigned)blocks, (unsigned)n_tensors);
    k_permute<<<grid, t, 0, s>>>((const uint4*)q, (const uint4*)k, (const uint4*)v, (uint4*)qp, (uint4*)kp,
                                 (uint4*)vp, p.d_perm, (int)p.N, p.H, vec_per_row, npad, total);
    return cudaGetLastError();
}

}  // namespace bsa
