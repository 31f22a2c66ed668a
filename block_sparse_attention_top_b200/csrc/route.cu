// Top-p block routing kernels (FVAttn review, section 3 "Stage 1: Sparse Mask
// Routing" and section 3.1; alanhou.org blog, "Key Concepts": Top-p routing with
// a Top-k safety floor; L_h from the review's Eq. 1).
//
//   k_pool       gather through the token order + block mean of Q and K (HBM bound)
//   k_scores     s_ij = <Qbar_i, Kbar_j> / sqrt(d), fp64 tiles
//   k_route_rows softmax, sort by (P desc, j asc), cumulative mass, Top-p cut,
//                Top-k floor -> count and importance order per row
//   k_csr_scan   exclusive scan of the counts -> row_ptr, nnz, L_h
//   k_csr_fill   copy each row's kept columns into col_idx
//
// Precision: pooled sums are accumulated in fp64 (bf16 values sum exactly),
// scores, softmax and the cumulative mass are fp64, so the mask decision is
// stable far below the 1e-6 relative tie tolerance the kernels are held to.
#include <cuda_bf16.h>
#include <math.h>

#include "bsa_internal.cuh"

namespace bsa {
namespace {

// ---------------------------------------------------------------------------
// Pooling: one CTA per (query/key tensor, batch, block, chunk of the H*d row).
// Each thread owns 8 (bf16) or 4 (fp32) consecutive elements of a token row
// (one 16-byte load per token) and sums them over the block's tokens.
// ---------------------------------------------------------------------------
constexpr int kPoolThreads = 256;
constexpr int kPoolUnroll = 8;

template <typename T> struct Vec16;
template <> struct Vec16<__nv_bfloat16> {
    static constexpr int n = 8;
    __device__ static void widen(const uint4& u, double* out) {
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            out[2 * e] = (double)__uint_as_float(w[e] << 16);
            out[2 * e + 1] = (double)__uint_as_float(w[e] & 0xFFFF0000u);
        }
    }
};
template <> struct Vec16<float> {
    static constexpr int n = 4;
    __device__ static void widen(const uint4& u, double* out) {
        out[0] = (double)__uint_as_float(u.x);
        out[1] = (double)__uint_as_float(u.y);
        out[2] = (double)__uint_as_float(u.z);
        out[3] = (double)__uint_as_float(u.w);
    }
};

template <typename T>
__global__ void __launch_bounds__(kPoolThreads)
k_pool(const T* __restrict__ q, const T* __restrict__ k, const int32_t* __restrict__ perm,
       double* __restrict__ qbar, double* __restrict__ kbar, int N, int H, int d, int block, int nb) {
    constexpr int V = Vec16<T>::n;
    __shared__ int32_t s_tok[128];
    const int i = blockIdx.x;
    const int which = blockIdx.z & 1;
    const int b = blockIdx.z >> 1;
    const T* x = which ? k : q;
    double* out = which ? kbar : qbar;
    const int lo = i * block;
    const int m = min(N, lo + block) - lo;
    for (int t = threadIdx.x; t < m; t += blockDim.x) s_tok[t] = perm[lo + t];
    __syncthreads();

    const int hd = H * d;
    const int c = blockIdx.y * blockDim.x + threadIdx.x;   // 16-byte chunk within the row
    if (c * V >= hd) return;
    const uint4* base = reinterpret_cast<const uint4*>(x + (size_t)b * N * hd) + c;
    const size_t row_stride = (size_t)hd / V;              // in uint4

    double acc[V];
#pragma unroll
    for (int e = 0; e < V; ++e) acc[e] = 0.0;
    int t = 0;
    for (; t + kPoolUnroll <= m; t += kPoolUnroll) {
        uint4 u[kPoolUnroll];
#pragma unroll
        for (int r = 0; r < kPoolUnroll; ++r) u[r] = __ldg(base + (size_t)s_tok[t + r] * row_stride);
#pragma unroll
        for (int r = 0; r < kPoolUnroll; ++r) {
            double w[V];
            Vec16<T>::widen(u[r], w);
#pragma unroll
            for (int e = 0; e < V; ++e) acc[e] += w[e];
        }
    }
    for (; t < m; ++t) {
        const uint4 u = __ldg(base + (size_t)s_tok[t] * row_stride);
        double w[V];
        Vec16<T>::widen(u, w);
#pragma unroll
        for (int e = 0; e < V; ++e) acc[e] += w[e];
    }
    const int h = (c * V) / d;
    const int dd = (c * V) % d;
    double* dst = out + (((size_t)b * H + h) * nb + i) * d + dd;
    const double md = (double)m;
#pragma unroll
    for (int e = 0; e < V; ++e) dst[e] = acc[e] / md;
}

// ---------------------------------------------------------------------------
// Scores: 64x64 output tile per CTA, 256 threads x (4x4) outputs, fp64 FMA,
// d consumed in slices of 16 through shared memory.
// ---------------------------------------------------------------------------
constexpr int kST = 64, kSK = 16;

__global__ void __launch_bounds__(256)
k_scores(const double* __restrict__ qbar, const double* __restrict__ kbar, double* __restrict__ S,
         int nb, int d, double scale) {
    __shared__ double As[kSK][kST + 1];
    __shared__ double Bs[kSK][kST + 1];
    const int bh = blockIdx.z;
    const int i0 = blockIdx.y * kST, j0 = blockIdx.x * kST;
    const double* Q = qbar + (size_t)bh * nb * d;
    const double* K = kbar + (size_t)bh * nb * d;
    const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
    double acc[4][4] = {};
    for (int k0 = 0; k0 < d; k0 += kSK) {
        for (int e = threadIdx.x; e < kST * kSK; e += 256) {
            const int r = e / kSK, kk = e % kSK;
            As[kk][r] = (i0 + r < nb) ? Q[(size_t)(i0 + r) * d + k0 + kk] : 0.0;
            Bs[kk][r] = (j0 + r < nb) ? K[(size_t)(j0 + r) * d + k0 + kk] : 0.0;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < kSK; ++kk) {
            double a[4], bv[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) { a[u] = As[kk][ty + 16 * u]; bv[u] = Bs[kk][tx + 16 * u]; }
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int v = 0; v < 4; ++v) acc[u][v] = fma(a[u], bv[v], acc[u][v]);
        }
        __syncthreads();
    }
    double* out = S + (size_t)bh * nb * nb;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int i = i0 + ty + 16 * u;
        if (i >= nb) continue;
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            const int j = j0 + tx + 16 * v;
            if (j < nb) out[(size_t)i * nb + j] = acc[u][v] * scale;
        }
    }
}

// ---------------------------------------------------------------------------
// Row routing: one CTA per row.  The row's scores are sorted in shared memory
// by (s desc, j asc) -- softmax is monotone, so this is the order of P -- with
// a bitonic network over the next power of two; then P_(n), the inclusive
// cumulative mass, and the smallest n with C_n >= p.
// ---------------------------------------------------------------------------
constexpr int kRouteThreads = 256;

__device__ __forceinline__ bool before(double sa, int ja, double sb, int jb) {
    return sa > sb || (sa == sb && ja < jb);
}

template <typename Op>
__device__ double block_reduce(double v, double* red, Op op) {
    for (int o = 16; o > 0; o >>= 1) v = op(v, __shfl_xor_sync(0xffffffffu, v, o));
    const int w = threadIdx.x / 32, l = threadIdx.x % 32;
    __syncthreads();
    if (l == 0) red[w] = v;
    __syncthreads();
    v = red[0];
    for (int u = 1; u < (int)(blockDim.x / 32); ++u) v = op(v, red[u]);
    return v;
}

__global__ void __launch_bounds__(kRouteThreads)
k_route_rows(const double* __restrict__ S, int nb, int nbp, double p, int k_floor,
             uint16_t* __restrict__ sorted, int32_t* __restrict__ counts) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    double* key = reinterpret_cast<double*>(smem_raw);            // [nbp]
    int* idx = reinterpret_cast<int*>(key + nbp);                 // [nbp]
    __shared__ double red[kRouteThreads / 32];
    __shared__ double wsum[kRouteThreads / 32];
    __shared__ int s_np;
    const size_t r = blockIdx.x;
    const double* row = S + r * nb;
    const int tid = threadIdx.x;

    double mx = -INFINITY;
    for (int j = tid; j < nbp; j += blockDim.x) {
        const double s = j < nb ? row[j] : -INFINITY;
        key[j] = s;
        idx[j] = j;
        mx = fmax(mx, s);
    }
    mx = block_reduce(mx, red, [](double a, double b) { return fmax(a, b); });
    double z = 0.0;
    for (int j = tid; j < nb; j += blockDim.x) z += exp(key[j] - mx);
    z = block_reduce(z, red, [](double a, double b) { return a + b; });

    // bitonic sort, "before" order first
    for (int size = 2; size <= nbp; size <<= 1) {
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            __syncthreads();
            for (int t = tid; t < nbp / 2; t += blockDim.x) {
                const int a = 2 * t - (t & (stride - 1));
                const int b = a + stride;
                const bool up = (a & size) == 0;       // this half sorts in "before" order
                const double ka = key[a], kb = key[b];
                const int ia = idx[a], ib = idx[b];
                const bool swap = up ? before(kb, ib, ka, ia) : before(ka, ia, kb, ib);
                if (swap) { key[a] = kb; key[b] = ka; idx[a] = ib; idx[b] = ia; }
            }
        }
    }
    __syncthreads();

    // P in sorted order, inclusive scan: each thread owns a contiguous run
    const int per = (nbp + blockDim.x - 1) / blockDim.x;
    const int lo = tid * per, hi = min(nb, lo + per);
    double run = 0.0;
    for (int n = lo; n < hi; ++n) { const double pn = exp(key[n] - mx) / z; run += pn; key[n] = run; }
    // exclusive scan of per-thread totals
    double incl = run;
    const int lane = tid % 32, wid = tid / 32;
    for (int o = 1; o < 32; o <<= 1) {
        const double y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) wsum[wid] = incl;
    if (tid == 0) s_np = nb;
    __syncthreads();
    double off = incl - run;
    for (int w = 0; w < wid; ++w) off += wsum[w];
    int first = nb;
    for (int n = lo; n < hi; ++n) {
        const double c = key[n] + off;
        if (c >= p) { first = n + 1; break; }
    }
    if (first < nb) atomicMin(&s_np, first);
    __syncthreads();
    int n_p = s_np;
    if (p >= 1.0) n_p = nb;
    const int n_i = min(nb, max(k_floor, n_p));
    uint16_t* dst = sorted + r * nb;
    for (int n = tid; n < n_i; n += blockDim.x) dst[n] = (uint16_t)idx[n];
    if (tid == 0) counts[r] = n_i;
}

// ---------------------------------------------------------------------------
// CSR: single-CTA exclusive scan of the counts, then a row-parallel copy.
// ---------------------------------------------------------------------------
constexpr int kScanThreads = 1024;

__global__ void __launch_bounds__(kScanThreads)
k_csr_scan(const int32_t* __restrict__ counts, int64_t rows, int nb, int32_t* __restrict__ row_ptr,
           float* __restrict__ L_h, int64_t* __restrict__ nnz, int64_t col_cap, int32_t* err) {
    __shared__ long long wsum[kScanThreads / 32];
    const int tid = threadIdx.x;
    const int64_t per = (rows + kScanThreads - 1) / kScanThreads;
    const int64_t lo = tid * per, hi = min(rows, lo + per);
    long long run = 0;
    for (int64_t r = lo; r < hi; ++r) run += counts[r];
    long long incl = run;
    const int lane = tid % 32, wid = tid / 32;
    for (int o = 1; o < 32; o <<= 1) {
        const long long y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) wsum[wid] = incl;
    __syncthreads();
    long long off = incl - run;
    for (int w = 0; w < wid; ++w) off += wsum[w];
    for (int64_t r = lo; r < hi; ++r) {
        row_ptr[r] = (int32_t)off;
        off += counts[r];
    }
    if (tid == kScanThreads - 1) {
        row_ptr[rows] = (int32_t)off;
        *nnz = off;
        if (off > col_cap) record_error(err, BSA_ECAPACITY, 0);
    }
    __syncthreads();
    // L_h: integer sum over a head's rows, then one fp32 divide (Eq. 1)
    const int64_t heads = rows / nb;
    for (int64_t bh = tid; bh < heads; bh += kScanThreads)
        L_h[bh] = (float)(row_ptr[(bh + 1) * nb] - row_ptr[bh * nb]) / (float)nb;
}

__global__ void k_csr_fill(const int32_t* __restrict__ counts, const uint16_t* __restrict__ sorted,
                           const int32_t* __restrict__ row_ptr, int32_t* __restrict__ col_idx,
                           int64_t rows, int nb, int64_t col_cap) {
    const int64_t r = (int64_t)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
    if (r >= rows) return;
    const int n = counts[r];
    const int64_t base = row_ptr[r];
    const uint16_t* src = sorted + r * nb;
    for (int t = threadIdx.x % 32; t < n; t += 32)
        if (base + t < col_cap) col_idx[base + t] = src[t];
}

}  // namespace

cudaError_t launch_pool(const bsa_plan& p, const void* q, const void* k, int dtype,
                        double* qbar, double* kbar, cudaStream_t s) {
    const int V = dtype == BSA_BF16 ? 8 : 4;
    const int chunks = (p.H * p.d) / V;
    dim3 grid((unsigned)p.nb, (unsigned)((chunks + kPoolThreads - 1) / kPoolThreads), (unsigned)(2 * p.B));
    if (dtype == BSA_BF16)
        k_pool<__nv_bfloat16><<<grid, kPoolThreads, 0, s>>>((const __nv_bfloat16*)q, (const __nv_bfloat16*)k,
                                                           p.d_perm, qbar, kbar, (int)p.N, p.H, p.d, p.block, (int)p.nb);
    else
        k_pool<float><<<grid, kPoolThreads, 0, s>>>((const float*)q, (const float*)k, p.d_perm, qbar, kbar,
                                                   (int)p.N, p.H, p.d, p.block, (int)p.nb);
    return cudaGetLastError();
}

cudaError_t launch_scores(const bsa_plan& p, const double* qbar, const double* kbar, double* scores,
                          cudaStream_t s) {
    const int t = (int)((p.nb + kST - 1) / kST);
    dim3 grid(t, t, (unsigned)(p.B * p.H));
    k_scores<<<grid, 256, 0, s>>>(qbar, kbar, scores, (int)p.nb, p.d, 1.0 / sqrt((double)p.d));
    return cudaGetLastError();
}

cudaError_t launch_route_rows(const bsa_plan& p, const double* scores, double pval, int k_floor,
                              uint16_t* sorted, int32_t* counts, cudaStream_t s) {
    int nbp = 1;
    while (nbp < p.nb) nbp <<= 1;
    nbp = nbp < 2 ? 2 : nbp;
    const size_t smem = (size_t)nbp * (sizeof(double) + sizeof(int));
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(k_route_rows, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    k_route_rows<<<(unsigned)p.rows, kRouteThreads, smem, s>>>(scores, (int)p.nb, nbp, pval, k_floor, sorted, counts);
    return cudaGetLastError();
}

cudaError_t launch_csr(const bsa_plan& p, const int32_t* counts, const uint16_t* sorted, int32_t* row_ptr,
                       int32_t* col_idx, int64_t col_cap, float* L_h, int64_t* nnz, cudaStream_t s) {
    k_csr_scan<<<1, kScanThreads, 0, s>>>(counts, p.rows, (int)p.nb, row_ptr, L_h, nnz, col_cap, p.d_err);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (col_cap == 0) return cudaSuccess;
    const int rows_per_cta = 8;
    k_csr_fill<<<(unsigned)((p.rows + rows_per_cta - 1) / rows_per_cta), 32 * rows_per_cta, 0, s>>>(
        counts, sorted, row_ptr, col_idx, p.rows, (int)p.nb, col_cap);
    return cudaGetLastError();
}

}  // namespace bsa
