// Attention preparation: the work list and the reordered, zero-padded Q/K/V
// tiles.
//
// Work list: the order in which the persistent attention kernel's CTAs take
// the items (b, h, i) -- the single-GPU counterpart of the pages' runtime load
// balancing (FVAttn review, section 3.2: the heavy heads set the critical
// path), which here balances the kernel's CTAs instead of ranks.  Three
// schedules (bsa_plan_set_schedule):
//   BSA_SCHED_L2_HEADS        heads in groups whose K and V tiles fit a share
//                             of L2, groups by descending total work, items of
//                             a group by descending count: the CTAs that run
//                             at the same time read the same few heads' tiles,
//                             so those tiles are served from L2 (default);
//   BSA_SCHED_HEAVIEST_FIRST  every item by descending count (longest
//                             processing time first over all heads);
//   BSA_SCHED_IN_ORDER        items in row order.
// The sorted schedules are one counting sort on an ascending position key
// (histogram, exclusive scan, scatter); the order among items with equal keys
// is unspecified (it does not change results).
//
// Permutation: Xp[b, h, n', :] = X[b, perm[n'], h, :] for n' < N and zero for
// the padding rows N <= n' < nb*block (FVAttn review, section 3.1: Hilbert
// curve block reordering), so every key/value block is one dense
// [block, d] tile the attention kernel can fetch with a single TMA box.
#include <cuda_bf16.h>

#include <algorithm>

#include "bsa_internal.cuh"

namespace bsa {
namespace {

// Rank of each head group by descending total work (ties: lower group first).
// One CTA; a group is heads [g*G, (g+1)*G) and its rows are contiguous.
__global__ void k_group_rank(const int32_t* __restrict__ row_ptr, int64_t rows, int64_t rows_per_group,
                             int groups, int32_t* __restrict__ grank) {
    extern __shared__ long long gw[];
    for (int g = threadIdx.x; g < groups; g += blockDim.x) {
        const int64_t lo = (int64_t)g * rows_per_group, hi = min(rows, lo + rows_per_group);
        gw[g] = (long long)row_ptr[hi] - (long long)row_ptr[lo];
    }
    __syncthreads();
    for (int g = threadIdx.x; g < groups; g += blockDim.x) {
        const long long wg = gw[g];
        int rank = 0;
        for (int u = 0; u < groups; ++u) rank += (gw[u] > wg || (gw[u] == wg && u < g)) ? 1 : 0;
        grank[g] = rank;
    }
}

// Position key of row r: bins are visited in ascending key order.
struct SchedKey {
    int nb;
    int64_t rows_per_group;
    const int32_t* grank;       // null: one group (plain heaviest-first)
    __device__ int operator()(int64_t r, int n) const {
        const int within = nb - n;                              // larger counts first
        return grank ? grank[r / rows_per_group] * (nb + 1) + within : within;
    }
};

__device__ __forceinline__ int row_count(const int32_t* row_ptr, int64_t r, int nb, int32_t* err) {
    int n = row_ptr[r + 1] - row_ptr[r];
    if (n < 0 || n > nb) {                       // malformed mask: record, clamp
        if (err) record_error(err, BSA_EDEVICE, (int)r);
        n = n < 0 ? 0 : nb;
    }
    return n;
}

__global__ void k_hist(const int32_t* __restrict__ row_ptr, int64_t rows, SchedKey key,
                       int32_t* __restrict__ hist, int32_t* err) {
    const int64_t r = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (r >= rows) return;
    atomicAdd(&hist[key(r, row_count(row_ptr, r, key.nb, err))], 1);
}

// bins[u] = number of items whose key is below u (exclusive scan).  One CTA.
__global__ void k_bins(const int32_t* __restrict__ hist, int n_bins, int32_t* __restrict__ bins) {
    __shared__ int wsum[32];
    const int tid = threadIdx.x;
    const int per = (n_bins + blockDim.x - 1) / blockDim.x;
    const int lo = min(n_bins, tid * per), hi = min(n_bins, lo + per);
    int run = 0;
    for (int u = lo; u < hi; ++u) run += hist[u];
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
        bins[u] = off;
        off += hist[u];
    }
}

__global__ void k_scatter(const int32_t* __restrict__ row_ptr, int64_t rows, SchedKey key,
                          int32_t* __restrict__ bins, int32_t* __restrict__ work) {
    const int64_t r = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (r >= rows) return;
    const int pos = atomicAdd(&bins[key(r, row_count(row_ptr, r, key.nb, nullptr))], 1);
    work[pos] = (int32_t)r;
}

// In-order schedule: work[r] = r (the counts are still checked).
__global__ void k_iota(const int32_t* __restrict__ row_ptr, int64_t rows, int nb, int32_t* __restrict__ work,
                       int32_t* err) {
    const int64_t r = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (r >= rows) return;
    row_count(row_ptr, r, nb, err);
    work[r] = (int32_t)r;
}

// One CTA per kPermRows consecutive destination rows n of the padded sequence
// (and batch entry, tensor): each row copies token perm[n]'s contiguous H*d row
// into the H per-head tiles (zeros for the padding rows n >= N).  Thread t moves
// the 16-byte chunks t, t + blockDim, ... of the row, the loads of the CTA's
// rows in flight together; a head's rows land as one contiguous run.
constexpr int kPermRows = 4;

__global__ void __launch_bounds__(1024)
k_permute(const uint4* __restrict__ q, const uint4* __restrict__ k, const uint4* __restrict__ v,
          uint4* __restrict__ qp, uint4* __restrict__ kp, uint4* __restrict__ vp, const int32_t* __restrict__ perm,
          int N, int H, int vec_per_row, int64_t npad) {
    const int b = blockIdx.y;
    const uint4* src = blockIdx.z == 0 ? q : (blockIdx.z == 1 ? k : v);
    uint4* dst = blockIdx.z == 0 ? qp : (blockIdx.z == 1 ? kp : vp);
    const int row_vecs = H * vec_per_row;
    int64_t n[kPermRows], srow[kPermRows];
    bool real[kPermRows];
#pragma unroll
    for (int r = 0; r < kPermRows; ++r) {
        n[r] = (int64_t)blockIdx.x * kPermRows + r;
        real[r] = n[r] < N;
        srow[r] = real[r] ? ((int64_t)b * N + perm[n[r]]) * row_vecs : 0;
    }
    for (int e = threadIdx.x; e < row_vecs; e += blockDim.x) {
        const int h = e / vec_per_row, c = e - h * vec_per_row;
        uint4 val[kPermRows];
#pragma unroll
        for (int r = 0; r < kPermRows; ++r) val[r] = real[r] ? __ldg(src + srow[r] + e) : make_uint4(0u, 0u, 0u, 0u);
        uint4* out = dst + ((int64_t)b * H + h) * npad * vec_per_row + c;
#pragma unroll
        for (int r = 0; r < kPermRows; ++r)
            if (n[r] < npad) out[n[r] * vec_per_row] = val[r];
    }
}

}  // namespace

int sched_heads_per_group(const bsa_plan& p) {
    // K and V tiles of one head: 2 * nb * block * d bf16 values
    const double head_bytes = 2.0 * (double)p.nb * p.block * p.d * 2.0;
    const double budget = 0.4 * (double)p.l2_bytes;
    const int g = (int)(budget / head_bytes);
    return g < 1 ? 1 : (g > p.B * p.H ? p.B * p.H : g);
}

int64_t sched_bins(const bsa_plan& p) {
    const int64_t heads = (int64_t)p.B * p.H;
    return (heads + 1) * (p.nb + 1);
}

cudaError_t launch_worklist(const bsa_plan& p, const int32_t* row_ptr, int32_t* hist, int32_t* bins,
                            int32_t* grank, int32_t* work, cudaStream_t s) {
    const int t = 256;
    const unsigned g = (unsigned)((p.rows + t - 1) / t);
    if (p.schedule == BSA_SCHED_IN_ORDER) {
        k_iota<<<g, t, 0, s>>>(row_ptr, p.rows, (int)p.nb, work, p.d_err);
        return cudaGetLastError();
    }
    SchedKey key{(int)p.nb, p.rows, nullptr};
    int n_bins = (int)p.nb + 1;
    const int G = sched_heads_per_group(p);
    const int groups = (int)((p.B * p.H + G - 1) / G);
    if (p.schedule == BSA_SCHED_L2_HEADS && groups > 1 && groups <= kMaxSchedGroups) {
        key.rows_per_group = (int64_t)G * p.nb;
        key.grank = grank;
        n_bins = groups * ((int)p.nb + 1);
        const size_t smem = (size_t)groups * sizeof(long long);
        if (smem > 48 * 1024) {
            cudaError_t e = cudaFuncSetAttribute(k_group_rank, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            if (e != cudaSuccess) return e;
        }
        k_group_rank<<<1, 1024, smem, s>>>(row_ptr, p.rows, key.rows_per_group, groups, grank);
    }
    cudaError_t e = cudaMemsetAsync(hist, 0, (size_t)n_bins * sizeof(int32_t), s);
    if (e != cudaSuccess) return e;
    k_hist<<<g, t, 0, s>>>(row_ptr, p.rows, key, hist, p.d_err);
    k_bins<<<1, 1024, 0, s>>>(hist, n_bins, bins);
    k_scatter<<<g, t, 0, s>>>(row_ptr, p.rows, key, bins, work);
    return cudaGetLastError();
}

cudaError_t launch_permute(const bsa_plan& p, const void* q, const void* k, const void* v, void* qp,
                           void* kp, void* vp, cudaStream_t s, int n_tensors) {
    const int vec_per_row = p.d * 2 / 16;
    const int64_t npad = p.nb * p.block;
    const int row_vecs = p.H * vec_per_row;
    const int t = std::min(1024, (row_vecs + 31) / 32 * 32);
    const dim3 grid((unsigned)((npad + kPermRows - 1) / kPermRows), (unsigned)p.B, (unsigned)n_tensors);
    k_permute<<<grid, t, 0, s>>>((const uint4*)q, (const uint4*)k, (const uint4*)v, (uint4*)qp, (uint4*)kp,
                                 (uint4*)vp, p.d_perm, (int)p.N, p.H, vec_per_row, npad);
    return cudaGetLastError();
}

}  // namespace bsa
