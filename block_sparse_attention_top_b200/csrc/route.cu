// Top-p block routing kernels (FVAttn review, section 3 "Stage 1: Sparse Mask
// Routing" and section 3.1; alanhou.org blog, "Key Concepts": Top-p routing with
// a Top-k safety floor; L_h from the review's Eq. 1).
//
//   k_pool       gather through the token order + block mean of Q and K (HBM bound)
//   k_scores_mma s_ij = <Qbar_i, Kbar_j> / sqrt(d), fp64 MMA (m8n8k4)
//   k_route_warp   softmax, sort by (P desc, j asc), cumulative mass, Top-p
//   k_route_bwarp  cut, Top-k floor -> count and importance order per row
//   k_route_bucket (a register bitonic sort per warp up to 256 blocks, an
//   k_route_cta    exact bucket sort per warp up to 1024 and per CTA up to
//                  4096, a CTA bitonic sort above)
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

// The heads a launch covers: h0 .. h0 + nh - 1 of every batch entry.  Local
// head t (0 <= t < B * nh) is (b, h) = (t / nh, h0 + t % nh); local row l of
// a launch over rows is (local head l / nb, query block l % nb).
struct HeadRange {
    int H, h0, nh;
    __device__ __forceinline__ int bh(int t) const { return (t / nh) * H + h0 + t % nh; }
    // rows of a launch fit int32 (the library rejects rows * nb >= 2^31), so 32-bit division
    __device__ __forceinline__ int64_t row(int64_t l, int nb) const {
        const int l32 = (int)l, t = l32 / nb;
        return (int64_t)bh(t) * nb + (l32 - t * nb);
    }
};

// ---------------------------------------------------------------------------
// Pooling: one CTA per (block, query/key tensor and batch entry, share of the
// H*d row).  Thread c owns the 16-byte chunk c of a token row (8 bf16 or 4 fp32
// values) and sums it over every token of the block, 16 loads in flight, so
// the CTAs of a block read whole token rows from DRAM (measured 18 % faster
// than CTAs that each gathered a 1 KB slice of the rows).  Sums of bf16 (or
// fp32) values in fp64 are exact here, so the summation order does not change
// the result.
// ---------------------------------------------------------------------------
constexpr int kPoolTarget = 320;             // threads per CTA the row shares aim at
constexpr int kPoolUnroll = 16;

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
__global__ void __launch_bounds__(1024, 1)
k_pool(const T* __restrict__ q, const T* __restrict__ k, const int32_t* __restrict__ perm,
       double* __restrict__ qbar, double* __restrict__ kbar, int N, int H, int d, int block, int nb, int chunk0,
       int chunk_end) {
    constexpr int V = Vec16<T>::n;
    __shared__ int32_t s_tok[128];
    const int i = blockIdx.x, which = blockIdx.y & 1, b = blockIdx.y >> 1;
    const T* x = which ? k : q;
    double* out = which ? kbar : qbar;
    const int lo = i * block;
    const int m = min(N, lo + block) - lo;
    for (int t = threadIdx.x; t < m; t += blockDim.x) s_tok[t] = perm[lo + t];
    __syncthreads();
    const int hd = H * d;
    const size_t row_stride = (size_t)hd / V;              // in uint4
    for (int c = chunk0 + blockIdx.z * blockDim.x + threadIdx.x; c < chunk_end; c += blockDim.x * gridDim.z) {
        const uint4* base = reinterpret_cast<const uint4*>(x + (size_t)b * N * hd) + c;
        double acc[V];
#pragma unroll
        for (int e = 0; e < V; ++e) acc[e] = 0.0;
        int t = 0;
        for (; t + kPoolUnroll <= m; t += kPoolUnroll) {
            uint4 u[kPoolUnroll];
#pragma unroll
            for (int r = 0; r < kPoolUnroll; ++r) u[r] = __ldg(base + (size_t)s_tok[t + r] * row_stride);
            asm volatile("" ::: "memory");          // every load of the batch is issued before any is used
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
}

// ---------------------------------------------------------------------------
// Scores on the FP64 MMA path (mma.sync m8n8k4 .f64: fp64 products and sums).
// CTA tile 64 x 64 of one head, 4 warps of 32 x 32 (4 x 4 tiles of 8 x 8);
// Qbar and Kbar staged by cp.async in slices of 16 along d, double-buffered.  Fragments
// of m8n8k4: A (8x4) a0 = A[lane/4][lane%4]; B (4x8) b0 = B[lane%4][lane/4];
// C (8x8) c0, c1 = C[lane/4][2*(lane%4) + {0,1}].
// ---------------------------------------------------------------------------
constexpr int kMT = 64;                  // CTA tile (rows and columns)
constexpr int kMK = 16;                  // d slice
constexpr int kMLd = kMK + 4;            // shared row of 20 doubles: a half-warp's fragment reads
                                         // (rows g, columns t) and 16-byte stores hit distinct banks

__device__ __forceinline__ void dmma(double& c0, double& c1, double a, double b) {
    asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0,%1}, {%2}, {%3}, {%0,%1};"
                 : "+d"(c0), "+d"(c1)
                 : "d"(a), "d"(b));
}

__global__ void __launch_bounds__(128, 4)
k_scores_mma(const double* __restrict__ qbar, const double* __restrict__ kbar, double* __restrict__ S, int nb,
             int d, double scale, HeadRange hr) {
    __shared__ __align__(16) double As[2][kMT][kMLd];
    __shared__ __align__(16) double Bs[2][kMT][kMLd];
    const int bh = hr.bh(blockIdx.z);
    const int i0 = blockIdx.y * kMT, j0 = blockIdx.x * kMT;
    const double* Q = qbar + (size_t)bh * nb * d;
    const double* K = kbar + (size_t)bh * nb * d;
    const int tid = threadIdx.x, lane = tid % 32, warp = tid / 32;
    const int g = lane >> 2, t = lane & 3;
    const int wm = (warp >> 1) * 32, wn = (warp & 1) * 32;
    double acc[4][4][2];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b][0] = acc[a][b][1] = 0.0;
    // slices staged by cp.async (16 bytes per copy, zero-filled past nb): 64 rows x 16
    // doubles per operand = 512 copies, 4 per thread per operand
    auto issue = [&](int k0, int buf) {
#pragma unroll
        for (int l = 0; l < 4; ++l) {
            const int e = tid + 128 * l, r = e / (kMK / 2), c2 = e % (kMK / 2);
            const bool vq = i0 + r < nb, vk = j0 + r < nb;
            const double* gq = vq ? Q + (size_t)(i0 + r) * d + k0 + 2 * c2 : Q;
            const double* gk = vk ? K + (size_t)(j0 + r) * d + k0 + 2 * c2 : K;
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"((uint32_t)__cvta_generic_to_shared(&As[buf][r][2 * c2])),
                         "l"(gq), "r"(vq ? 16 : 0) : "memory");
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"((uint32_t)__cvta_generic_to_shared(&Bs[buf][r][2 * c2])),
                         "l"(gk), "r"(vk ? 16 : 0) : "memory");
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };
    const bool live = i0 + wm < nb && j0 + wn < nb;
    issue(0, 0);
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    __syncthreads();
    int buf = 0;
    for (int k0 = 0; k0 < d; k0 += kMK) {
        const bool more = k0 + kMK < d;
        if (more) issue(k0 + kMK, buf ^ 1);           // the other buffer was last read one slice ago
        if (live) {
#pragma unroll
            for (int ks = 0; ks < kMK / 4; ++ks) {
                double av[4], bv[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    av[u] = As[buf][wm + 8 * u + g][4 * ks + t];
                    bv[u] = Bs[buf][wn + 8 * u + g][4 * ks + t];
                }
#pragma unroll
                for (int mt = 0; mt < 4; ++mt)
#pragma unroll
                    for (int nt = 0; nt < 4; ++nt) dmma(acc[mt][nt][0], acc[mt][nt][1], av[mt], bv[nt]);
            }
        }
        asm volatile("cp.async.wait_group 0;" ::: "memory");
        __syncthreads();
        buf ^= 1;
    }
    double* out = S + (size_t)bh * nb * nb;
#pragma unroll
    for (int mt = 0; mt < 4; ++mt) {
        const int i = i0 + wm + 8 * mt + g;
        if (i >= nb) continue;
#pragma unroll
        for (int nt = 0; nt < 4; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int j = j0 + wn + 8 * nt + 2 * t + e;
                if (j < nb) out[(size_t)i * nb + j] = acc[mt][nt][e] * scale;
            }
    }
}

// ---------------------------------------------------------------------------
// Row routing, one warp per row (nb <= 1024).  Each lane holds E = nbp/32
// consecutive elements of the padded row as one 64-bit key that sorts in
// ascending order exactly as (s descending, j ascending): the order-preserving
// image of s, complemented, with its 13 lowest bits replaced by j.  (Dropping
// those bits only merges scores equal to ~1e-12 relative, far inside the 1e-6
// tie tolerance, and then orders them by ascending j as the exact rule does.)
// A bitonic network sorts the keys: exchanges between registers for strides
// below E, between lanes (shuffles) above.  P, the inclusive cumulative mass
// and the Top-p cut follow in fp64.
// ---------------------------------------------------------------------------
constexpr unsigned long long kJMask = 0x1FFFull;          // 13-bit block index field (nb <= 8192)
constexpr unsigned long long kPadKey = ~0ull & ~kJMask;    // sorts after every real score
__device__ __forceinline__ unsigned long long desc_key(double s, int j) {
    unsigned long long u = (unsigned long long)__double_as_longlong(s);
    u = (u & 0x8000000000000000ull) ? ~u : (u | 0x8000000000000000ull);   // ascending with s
    return (~u & ~kJMask) | (unsigned long long)j;
}
__device__ __forceinline__ double key_score(unsigned long long key) {
    unsigned long long u = ~(key | kJMask);                          // low bits of s are gone
    u = (u & 0x8000000000000000ull) ? (u & 0x7FFFFFFFFFFFFFFFull) : ~u;
    return __longlong_as_double((long long)u);
}

template <int E>
__global__ void __launch_bounds__(128, 1)
k_route_warp(const double* __restrict__ S, int64_t rows, int nb, double p, int k_floor,
             uint16_t* __restrict__ sorted, int32_t* __restrict__ counts, HeadRange hr) {
    constexpr int NBP = 32 * E;
    constexpr int LOGN = E == 1 ? 5 : E == 2 ? 6 : E == 4 ? 7 : E == 8 ? 8 : E == 16 ? 9 : 10;
    static_assert((1 << LOGN) == NBP, "E must be a power of two <= 32");
    const int lane = threadIdx.x % 32;
    const int64_t lr = (int64_t)blockIdx.x * 4 + threadIdx.x / 32;
    if (lr >= rows) return;
    const int64_t r = hr.row(lr, nb);
    const double* row = S + r * nb;
    unsigned long long key[E];
    double mx = -INFINITY;
#pragma unroll
    for (int k = 0; k < E; ++k) {
        const int e = lane * E + k;
        if (e < nb) {
            const double sv = row[e];
            mx = fmax(mx, sv);
            key[k] = desc_key(sv, e);
        } else {
            key[k] = kPadKey | (unsigned long long)(e & kJMask);               // after every score
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    double z = 0.0;
#pragma unroll
    for (int k = 0; k < E; ++k) z += (lane * E + k < nb) ? exp(key_score(key[k]) - mx) : 0.0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);

    // bitonic sort, ascending keys; every loop bound is a compile-time constant
#pragma unroll
    for (int ls = 1; ls <= LOGN; ++ls) {
#pragma unroll
        for (int lt = ls - 1; lt >= 0; --lt) {
            const int size = 1 << ls, stride = 1 << lt;
            if (stride < E) {
#pragma unroll
                for (int k = 0; k < E; ++k) {
                    if ((k & stride) == 0) {
                        const int kp = k | stride;
                        const bool up = ((lane * E + k) & size) == 0;
                        const unsigned long long a = key[k], b = key[kp];
                        const bool sw = up ? (b < a) : (a < b);
                        key[k] = sw ? b : a;
                        key[kp] = sw ? a : b;
                    }
                }
            } else {
                const int lmask = stride / E;
                const bool lower = (lane & lmask) == 0;
#pragma unroll
                for (int k = 0; k < E; ++k) {
                    const bool up = ((lane * E + k) & size) == 0;
                    const unsigned long long mine = key[k];
                    const unsigned long long other = __shfl_xor_sync(0xffffffffu, mine, lmask);
                    key[k] = ((other < mine) == (lower == up)) ? other : mine;
                }
            }
        }
    }
    // P in sorted order, inclusive cumulative mass, first n with C_n >= p
    double c[E];
    double run = 0.0;
#pragma unroll
    for (int k = 0; k < E; ++k) {
        const int e = lane * E + k;
        run += e < nb ? exp(key_score(key[k]) - mx) / z : 0.0;
        c[k] = run;
    }
    double excl = run;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const double y = __shfl_up_sync(0xffffffffu, excl, o);
        if (lane >= o) excl += y;
    }
    excl -= run;
    int first = nb;
#pragma unroll
    for (int k = E - 1; k >= 0; --k) {
        const int e = lane * E + k;
        if (e < nb && c[k] + excl >= p) first = e + 1;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) first = min(first, __shfl_xor_sync(0xffffffffu, first, o));
    const int n_p = p >= 1.0 ? nb : first;
    const int n_i = min(nb, max(k_floor, n_p));
    uint16_t* dst = sorted + r * nb;
#pragma unroll
    for (int k = 0; k < E; ++k) {
        const int e = lane * E + k;
        if (e < nb) dst[e] = (uint16_t)(key[k] & kJMask);     // the full importance order
    }
    if (lane == 0) counts[r] = n_i;
}

// ---------------------------------------------------------------------------
// Row routing for long rows (nbp >= 512): one 256-thread CTA per row, E =
// nbp/256 keys per thread (same keys as above).  Bitonic exchanges run inside
// a thread's registers for strides below E, by warp shuffle for strides below
// 32E, and through shared memory above (two barriers per such stage).
// ---------------------------------------------------------------------------
constexpr int kCtaSortThreads = 256;

template <int E>
__global__ void __launch_bounds__(kCtaSortThreads)
k_route_cta(const double* __restrict__ S, int nb, double p, int k_floor,
            uint16_t* __restrict__ sorted, int32_t* __restrict__ counts, HeadRange hr) {
    constexpr int NBP = kCtaSortThreads * E;
    constexpr int LOGN = E == 2 ? 9 : E == 4 ? 10 : E == 8 ? 11 : E == 16 ? 12 : 13;
    static_assert((1 << LOGN) == NBP, "E must be 2, 4, 8, 16 or 32");
    extern __shared__ unsigned long long xk[];              // [NBP] cross-warp exchange
    __shared__ double red[kCtaSortThreads / 32];
    __shared__ int s_first;
    const int tid = threadIdx.x, lane = tid % 32, wid = tid / 32;
    const size_t r = (size_t)hr.row(blockIdx.x, nb);
    const double* row = S + r * nb;
    unsigned long long key[E];
    double mx = -INFINITY;
#pragma unroll
    for (int k = 0; k < E; ++k) {
        const int e = tid * E + k;
        if (e < nb) {
            const double sv = row[e];
            mx = fmax(mx, sv);
            key[k] = desc_key(sv, e);
        } else {
            key[k] = kPadKey | (unsigned long long)(e & kJMask);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (lane == 0) red[wid] = mx;
    if (tid == 0) s_first = nb;
    __syncthreads();
    mx = red[0];
#pragma unroll
    for (int w = 1; w < kCtaSortThreads / 32; ++w) mx = fmax(mx, red[w]);
    double z = 0.0;
#pragma unroll
    for (int k = 0; k < E; ++k) z += (tid * E + k < nb) ? exp(key_score(key[k]) - mx) : 0.0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
    __syncthreads();                                         // everyone has read red[] (max)
    if (lane == 0) red[wid] = z;
    __syncthreads();
    z = 0.0;
#pragma unroll
    for (int w = 0; w < kCtaSortThreads / 32; ++w) z += red[w];

#pragma unroll
    for (int ls = 1; ls <= LOGN; ++ls) {
#pragma unroll
        for (int lt = ls - 1; lt >= 0; --lt) {
            const int size = 1 << ls, stride = 1 << lt;
            if (stride < E) {
#pragma unroll
                for (int k = 0; k < E; ++k) {
                    if ((k & stride) == 0) {
                        const int kp = k | stride;
                        const bool up = ((tid * E + k) & size) == 0;
                        const unsigned long long a = key[k], b = key[kp];
                        const bool sw = up ? (b < a) : (a < b);
                        key[k] = sw ? b : a;
                        key[kp] = sw ? a : b;
                    }
                }
            } else if (stride < 32 * E) {
                const int lmask = stride / E;
                const bool lower = (lane & lmask) == 0;
#pragma unroll
                for (int k = 0; k < E; ++k) {
                    const bool up = ((tid * E + k) & size) == 0;
                    const unsigned long long mine = key[k];
                    const unsigned long long other = __shfl_xor_sync(0xffffffffu, mine, lmask);
                    key[k] = ((other < mine) == (lower == up)) ? other : mine;
                }
            } else {
#pragma unroll
                for (int k = 0; k < E; ++k) xk[tid * E + k] = key[k];
                __syncthreads();
#pragma unroll
                for (int k = 0; k < E; ++k) {
                    const int e = tid * E + k;
                    const bool up = (e & size) == 0, lower = (e & stride) == 0;
                    const unsigned long long mine = key[k], other = xk[e ^ stride];
                    key[k] = ((other < mine) == (lower == up)) ? other : mine;
                }
                __syncthreads();
            }
        }
    }
    // P in sorted order, inclusive cumulative mass, first n with C_n >= p
    double c[E];
    double run = 0.0;
#pragma unroll
    for (int k = 0; k < E; ++k) {
        const int e = tid * E + k;
        run += e < nb ? exp(key_score(key[k]) - mx) / z : 0.0;
        c[k] = run;
    }
    double incl = run;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const double y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) red[wid] = incl;                        // red[] free: z was read before the sort
    __syncthreads();
    double excl = incl - run;
    for (int w = 0; w < wid; ++w) excl += red[w];
    int first = nb;
#pragma unroll
    for (int k = E - 1; k >= 0; --k) {
        const int e = tid * E + k;
        if (e < nb && c[k] + excl >= p) first = e + 1;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) first = min(first, __shfl_xor_sync(0xffffffffu, first, o));
    if (lane == 0 && first < nb) atomicMin(&s_first, first);
    __syncthreads();
    const int n_p = p >= 1.0 ? nb : s_first;
    const int n_i = min(nb, max(k_floor, n_p));
    uint16_t* dst = sorted + r * nb;
#pragma unroll
    for (int k = 0; k < E; ++k) {
        const int e = tid * E + k;
        if (e < nb) dst[e] = (uint16_t)(key[k] & kJMask);     // the full importance order
    }
    if (tid == 0) counts[r] = n_i;
}

// ---------------------------------------------------------------------------
// Row routing by an exact bucket sort (rows of more than 256 blocks): one
// 128-thread CTA per row.  Each score goes to bucket floor((max - s) * NB /
// (max - min)) -- monotone in s, so every key of a bucket sorts after every
// key of a lower bucket -- the buckets are laid out by a shared-memory count
// and exclusive scan, and each key takes its place inside its bucket by
// counting the smaller keys there (the same 64-bit keys as above: s
// descending, j ascending, so the result is the exact order).  P, the
// inclusive cumulative mass (a block scan in sorted order) and the Top-p cut
// follow in fp64, as in the warp kernel.
// ---------------------------------------------------------------------------
constexpr int kBucketThreads = 128;

__device__ __forceinline__ double block_sum(double v, double* red) {
    const int lane = threadIdx.x % 32, wid = threadIdx.x / 32;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    __syncthreads();
    if (lane == 0) red[wid] = v;
    __syncthreads();
    double t = 0.0;
#pragma unroll
    for (int w = 0; w < kBucketThreads / 32; ++w) t += red[w];
    return t;
}
__device__ __forceinline__ double block_max(double v, double* red) {
    const int lane = threadIdx.x % 32, wid = threadIdx.x / 32;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmax(v, __shfl_xor_sync(0xffffffffu, v, o));
    __syncthreads();
    if (lane == 0) red[wid] = v;
    __syncthreads();
    double t = red[0];
#pragma unroll
    for (int w = 1; w < kBucketThreads / 32; ++w) t = fmax(t, red[w]);
    return t;
}

// dynamic shared memory: keys [nb] u64, placed [nb] u64, pj [nb] f64 (exp(s_j - max)),
// bucket [nb] int, count [NB] int, start [NB] int
__global__ void __launch_bounds__(kBucketThreads)
k_route_bucket(const double* __restrict__ S, int nb, int NB, double p, int k_floor,
               uint16_t* __restrict__ sorted, int32_t* __restrict__ counts, HeadRange hr) {
    extern __shared__ unsigned long long bsm[];
    unsigned long long* keys = bsm;
    unsigned long long* placed = bsm + nb;
    double* pj = reinterpret_cast<double*>(bsm + 2 * nb);
    int* bucket = reinterpret_cast<int*>(bsm + 3 * nb);
    int* cnt = bucket + nb;
    int* start = cnt + NB;
    __shared__ double red[kBucketThreads / 32];
    __shared__ int wsum[kBucketThreads / 32];
    __shared__ int s_first;
    const int tid = threadIdx.x, lane = tid % 32, wid = tid / 32;
    const size_t r = (size_t)hr.row(blockIdx.x, nb);
    const double* row = S + r * nb;

    double mx = -INFINITY, mn = INFINITY;
    for (int j = tid; j < nb; j += kBucketThreads) {
        const double sv = row[j];
        mx = fmax(mx, sv);
        mn = fmin(mn, sv);
        keys[j] = desc_key(sv, j);
        pj[j] = sv;
    }
    for (int b = tid; b < NB; b += kBucketThreads) cnt[b] = 0;
    if (tid == 0) s_first = nb;
    mx = block_max(mx, red);
    mn = -block_max(-mn, red);
    const double width = mx - mn;
    const double to_bucket = width > 0.0 ? (double)NB / width : 0.0;
    // bucket of each score (monotone in s), the unnormalised mass exp(s - max) of its key
    double zpart = 0.0;
    for (int j = tid; j < nb; j += kBucketThreads) {
        const int b = min(NB - 1, (int)((mx - pj[j]) * to_bucket));
        bucket[j] = b;
        const double e = exp(key_score(keys[j]) - mx);
        pj[j] = e;
        zpart += e;
        atomicAdd(&cnt[b], 1);
    }
    const double z = block_sum(zpart, red);
    // exclusive scan of the counts (NB / 128 per thread, then across the block)
    {
        const int per = NB / kBucketThreads;
        const int lo = tid * per;
        int run = 0;
        for (int u = 0; u < per; ++u) run += cnt[lo + u];
        int incl = run;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        if (lane == 31) wsum[wid] = incl;
        __syncthreads();
        int off = incl - run;
        for (int w = 0; w < wid; ++w) off += wsum[w];
        for (int u = 0; u < per; ++u) {
            start[lo + u] = off;
            off += cnt[lo + u];
            cnt[lo + u] = 0;                      // reused as the fill cursor
        }
    }
    __syncthreads();
    for (int j = tid; j < nb; j += kBucketThreads) {
        const int b = bucket[j];
        placed[start[b] + atomicAdd(&cnt[b], 1)] = keys[j];
    }
    __syncthreads();
    // each key's final place: its bucket's start + the number of smaller keys in the bucket
    for (int q = tid; q < nb; q += kBucketThreads) {
        const unsigned long long key = placed[q];
        const int b = bucket[(int)(key & kJMask)];
        const int b0 = start[b], b1 = b0 + cnt[b];
        int rank = b0;
        for (int u = b0; u < b1; ++u) rank += placed[u] < key;
        keys[rank] = key;
    }
    __syncthreads();
    // P in sorted order, inclusive cumulative mass (contiguous chunks per thread), first n with C_n >= p
    const double inv_z = 1.0 / z;
    const int per = (nb + kBucketThreads - 1) / kBucketThreads;
    const int q0 = tid * per, q1 = min(nb, q0 + per);
    double run = 0.0;
    for (int q = q0; q < q1; ++q) run += pj[(int)(keys[q] & kJMask)] * inv_z;
    double incl = run;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const double y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) red[wid] = incl;
    __syncthreads();
    double c = incl - run;
    for (int w = 0; w < wid; ++w) c += red[w];
    int first = nb;
    for (int q = q0; q < q1; ++q) {
        c += pj[(int)(keys[q] & kJMask)] * inv_z;
        if (c >= p) { first = q + 1; break; }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) first = min(first, __shfl_xor_sync(0xffffffffu, first, o));
    if (lane == 0 && first < nb) atomicMin(&s_first, first);
    __syncthreads();
    const int n_p = p >= 1.0 ? nb : s_first;
    const int n_i = min(nb, max(k_floor, n_p));
    uint16_t* dst = sorted + r * nb;
    for (int q = tid; q < nb; q += kBucketThreads) dst[q] = (uint16_t)(keys[q] & kJMask);   // the full importance order
    if (tid == 0) counts[r] = n_i;
}

// ---------------------------------------------------------------------------
// Row routing by a warp-level exact bucket sort (rows of 257 to 1024 blocks):
// one warp per row, four rows per CTA, no CTA barrier.  Lane l keeps the keys
// of blocks l, l + 32, l + 64, ... in registers (the 64-bit keys above).  Each
// key goes to bucket floor((max - s) * NB / (max - min)), monotone in s,
// through a histogram of 16-bit counts in shared memory whose atomic add also
// returns the key's slot inside its bucket.  A warp scan turns the counts into
// bucket starts, the keys are scattered to their buckets, each key's rank is
// its bucket's start plus the number of smaller keys in the bucket, and the
// keys are rewritten in place in rank order.  The exponentials exp(s - max),
// their running sum in sorted order (a contiguous run of C keys per lane, C
// odd so that the lanes' 64-bit reads fall on distinct banks), the total z
// and the first n with sum_{k<=n} e_k >= p z follow in fp64.
// ---------------------------------------------------------------------------
constexpr int kBwarpRows = 4;

// Word of bucket pair w (buckets 2w, 2w + 1): one pad word after every NB / 64
// words, so that the lanes' contiguous ranges in the scan start on distinct banks.
__device__ __forceinline__ int bucket_word(int w, int NB) { return w + (w >> (__ffs(NB) - 7)); }
__device__ __forceinline__ int bucket_start(const uint32_t* bw, int b, int NB) {
    return (int)((bw[bucket_word(b >> 1, NB)] >> ((b & 1) * 16)) & 0xFFFFu);
}

// per-warp shared memory: keys [nb] u64, then NB / 2 + 33 words of two 16-bit
// counts (later starts; start[NB] = nb) with the pad words
__host__ __device__ __forceinline__ int bwarp_stride(int nb, int NB) { return nb + (NB / 2 + 34) / 2; }

template <int E>
__global__ void __launch_bounds__(32 * kBwarpRows)
k_route_bwarp(const double* __restrict__ S, int64_t rows, int nb, int NB, double p, int k_floor,
              uint16_t* __restrict__ sorted, int32_t* __restrict__ counts, HeadRange hr) {
    extern __shared__ unsigned long long wsm[];
    const int lane = threadIdx.x % 32, wid = threadIdx.x / 32;
    const int64_t lr = (int64_t)blockIdx.x * kBwarpRows + wid;
    if (lr >= rows) return;                               // the whole warp; nothing waits on it
    unsigned long long* keys = wsm + (size_t)wid * bwarp_stride(nb, NB);
    uint32_t* bw = reinterpret_cast<uint32_t*>(keys + nb);
    const int64_t r = hr.row(lr, nb);
    const double* row = S + r * nb;

    unsigned long long key[E];
    double mx = -INFINITY, mn = INFINITY;
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const int j = lane + 32 * e;
        key[e] = 0;
        if (j < nb) {
            key[e] = desc_key(row[j], j);
            const double sv = key_score(key[e]);
            mx = fmax(mx, sv);
            mn = fmin(mn, sv);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        mn = fmin(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    }
    for (int w = lane; w <= NB / 2 + 32; w += 32) bw[w] = 0;
    __syncwarp();
    // bucket of each key and its slot inside the bucket (arrival order, refined below)
    const double width = mx - mn;
    const double to_bucket = width > 0.0 ? (double)NB / width : 0.0;
    uint32_t slot[E];
#pragma unroll
    for (int e = 0; e < E; ++e) {
        slot[e] = 0;
        if (lane + 32 * e < nb) {
            const int b = min(NB - 1, (int)((mx - key_score(key[e])) * to_bucket));
            const int sh = (b & 1) * 16;
            const uint32_t old = atomicAdd(&bw[bucket_word(b >> 1, NB)], 1u << sh);
            slot[e] = (uint32_t)b | (((old >> sh) & 0xFFFFu) << 16);
        }
    }
    __syncwarp();
    // exclusive scan of the counts: lane l owns words [l (W + 1), l (W + 1) + W), W = NB / 64
    {
        const int W = NB / 64;
        uint32_t run = 0;
        for (int w = 0; w < W; ++w) {
            const uint32_t v = bw[lane * (W + 1) + w];
            run += (v & 0xFFFFu) + (v >> 16);
        }
        uint32_t incl = run;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        uint32_t off = incl - run;
        for (int w = 0; w < W; ++w) {
            const uint32_t v = bw[lane * (W + 1) + w];
            const uint32_t s0 = off, s1 = off + (v & 0xFFFFu);
            off = s1 + (v >> 16);
            bw[lane * (W + 1) + w] = s0 | (s1 << 16);
        }
        if (lane == 31) bw[bucket_word(NB / 2, NB)] = (uint32_t)nb;     // start[NB] = nb
    }
    __syncwarp();
#pragma unroll
    for (int e = 0; e < E; ++e)
        if (lane + 32 * e < nb) keys[bucket_start(bw, (int)(slot[e] & 0xFFFFu), NB) + (int)(slot[e] >> 16)] = key[e];
    __syncwarp();
    // each key's rank: its bucket's start + the smaller keys in the bucket
    int rk[E];
#pragma unroll
    for (int e = 0; e < E; ++e) {
        rk[e] = 0;
        if (lane + 32 * e < nb) {
            const int b = (int)(slot[e] & 0xFFFFu);
            const int b0 = bucket_start(bw, b, NB), b1 = bucket_start(bw, b + 1, NB);
            int rank = b0;
            for (int u = b0; u < b1; ++u) rank += keys[u] < key[e];
            rk[e] = rank;
        }
    }
    __syncwarp();
#pragma unroll
    for (int e = 0; e < E; ++e)
        if (lane + 32 * e < nb) keys[rk[e]] = key[e];
    __syncwarp();
    uint16_t* dst = sorted + r * nb;
    for (int q = lane; q < nb; q += 32) dst[q] = (uint16_t)(keys[q] & kJMask);   // the full importance order
    __syncwarp();
    // exponentials in sorted order (each lane a contiguous run of C keys, written over
    // its own keys), their running sum, then the Top-p cut
    const int C = ((nb + 31) / 32) | 1;
    const int q0 = min(nb, lane * C), q1 = min(nb, q0 + C);
    double* ex = reinterpret_cast<double*>(keys);
    double run = 0.0;
    for (int q = q0; q < q1; ++q) {
        const double e = exp(key_score(keys[q]) - mx);
        ex[q] = e;
        run += e;
    }
    double incl = run;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const double y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    const double target = p * __shfl_sync(0xffffffffu, incl, 31);
    double c = incl - run;
    int first = nb;
    for (int q = q0; q < q1; ++q) {
        c += ex[q];
        if (c >= target) {
            first = q + 1;
            break;
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) first = min(first, __shfl_xor_sync(0xffffffffu, first, o));
    const int n_p = p >= 1.0 ? nb : first;
    const int n_i = min(nb, max(k_floor, n_p));
    if (lane == 0) counts[r] = n_i;
}

// ---------------------------------------------------------------------------
// CSR: single-CTA exclusive scan of the counts, then a row-parallel copy.
// ---------------------------------------------------------------------------
constexpr int kScanThreads = 1024;

__global__ void __launch_bounds__(kScanThreads)
k_csr_scan(const int32_t* __restrict__ counts, int64_t rows, int nb, int32_t* __restrict__ row_ptr,
           float* __restrict__ L_h, int64_t* __restrict__ nnz, int64_t col_cap, int32_t* err) {
    // chunks of 4*kScanThreads rows (4 consecutive rows per thread): block-wide
    // scan of the per-thread sums, running offset carried between chunks
    __shared__ long long wsum[kScanThreads / 32];
    __shared__ long long s_carry;
    const int tid = threadIdx.x, lane = tid % 32, wid = tid / 32;
    if (tid == 0) s_carry = 0;
    __syncthreads();
    for (int64_t base = 0; base < rows; base += 4 * kScanThreads) {
        const int64_t r0 = base + 4 * (int64_t)tid;
        long long v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) v[u] = r0 + u < rows ? counts[r0 + u] : 0;
        const long long mine = v[0] + v[1] + v[2] + v[3];
        long long incl = mine;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const long long y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        if (lane == 31) wsum[wid] = incl;
        __syncthreads();
        long long off = s_carry + incl - mine;
        for (int w = 0; w < wid; ++w) off += wsum[w];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            if (r0 + u < rows) row_ptr[r0 + u] = (int32_t)off;
            off += v[u];
        }
        __syncthreads();                                   // all reads of wsum / s_carry done
        if (tid == kScanThreads - 1) s_carry = off;
        __syncthreads();
    }
    const long long total = s_carry;
    if (tid == 0) {
        row_ptr[rows] = (int32_t)total;
        *nnz = total;
        if (total > col_cap) record_error(err, BSA_ECAPACITY, 0);
    }
    __syncthreads();
    // L_h: integer sum over a head's rows, then one fp32 divide (Eq. 1)
    if (L_h == nullptr) return;
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
                        double* qbar, double* kbar, cudaStream_t s, int h0, int nh) {
    if (nh <= 0) nh = p.H - h0;
    const int V = dtype == BSA_BF16 ? 8 : 4;
    const int c0 = h0 * p.d / V, c1 = (h0 + nh) * p.d / V;     // chunks of heads h0 .. h0 + nh - 1
    const int split = (c1 - c0 + kPoolTarget - 1) / kPoolTarget;
    const int threads = ((c1 - c0 + split - 1) / split + 31) / 32 * 32;
    const dim3 grid((unsigned)p.nb, (unsigned)(2 * p.B), (unsigned)split);
    if (dtype == BSA_BF16)
        k_pool<__nv_bfloat16><<<grid, threads, 0, s>>>((const __nv_bfloat16*)q, (const __nv_bfloat16*)k, p.d_perm,
                                                       qbar, kbar, (int)p.N, p.H, p.d, p.block, (int)p.nb, c0, c1);
    else
        k_pool<float><<<grid, threads, 0, s>>>((const float*)q, (const float*)k, p.d_perm, qbar, kbar, (int)p.N,
                                               p.H, p.d, p.block, (int)p.nb, c0, c1);
    return cudaGetLastError();
}

cudaError_t launch_scores(const bsa_plan& p, const double* qbar, const double* kbar, double* scores,
                          cudaStream_t s, int h0, int nh) {
    if (nh <= 0) nh = p.H - h0;
    const double scale = 1.0 / sqrt((double)p.d);
    const int t = (int)((p.nb + kMT - 1) / kMT);            // d (64 or 128) is a multiple of the d slice
    dim3 grid(t, t, (unsigned)(p.B * nh));
    k_scores_mma<<<grid, 128, 0, s>>>(qbar, kbar, scores, (int)p.nb, p.d, scale, HeadRange{p.H, h0, nh});
    return cudaGetLastError();
}

cudaError_t launch_route_rows(const bsa_plan& p, const double* scores, double pval, int k_floor,
                              uint16_t* sorted, int32_t* counts, cudaStream_t s, int h0, int nh) {
    if (nh <= 0) nh = p.H - h0;
    const HeadRange hr{p.H, h0, nh};
    const int64_t rows = (int64_t)p.B * nh * p.nb;
    int nbp = 1;
    while (nbp < p.nb) nbp <<= 1;
    nbp = nbp < 2 ? 2 : nbp;
    const int nb = (int)p.nb;
    if (nbp <= 256) {
        const unsigned grid = (unsigned)((rows + 3) / 4);
        switch (nbp <= 32 ? 1 : nbp / 32) {
            case 1: k_route_warp<1><<<grid, 128, 0, s>>>(scores, rows, nb, pval, k_floor, sorted, counts, hr); break;
            case 2: k_route_warp<2><<<grid, 128, 0, s>>>(scores, rows, nb, pval, k_floor, sorted, counts, hr); break;
            case 4: k_route_warp<4><<<grid, 128, 0, s>>>(scores, rows, nb, pval, k_floor, sorted, counts, hr); break;
            default: k_route_warp<8><<<grid, 128, 0, s>>>(scores, rows, nb, pval, k_floor, sorted, counts, hr); break;
        }
        return cudaGetLastError();
    }
    if (nbp <= 1024) {
        // warp-level exact bucket sort: NB = 2 nbp buckets (2048 at 591 blocks: 12 us faster
        // than 512 there), E >= ceil(nb / 32) keys per lane (odd)
        const int NB = 2 * nbp;
        const size_t smem = (size_t)kBwarpRows * bwarp_stride(nb, NB) * sizeof(unsigned long long);
        const unsigned grid = (unsigned)((rows + kBwarpRows - 1) / kBwarpRows);
        const int need = ((nb + 31) / 32) | 1;
        auto run = [&](auto kern) -> cudaError_t {
            if (smem > 48 * 1024) {
                cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
                if (e != cudaSuccess) return e;
            }
            kern<<<grid, 32 * kBwarpRows, smem, s>>>(scores, rows, nb, NB, pval, k_floor, sorted, counts, hr);
            return cudaGetLastError();
        };
        if (need <= 13) return run(k_route_bwarp<13>);
        if (need <= 21) return run(k_route_bwarp<21>);
        return run(k_route_bwarp<33>);
    }
    if (nbp <= 4096) {
        // exact bucket sort: NB = nbp buckets (a multiple of the block size)
        const int NB = nbp;
        const size_t smem = (size_t)3 * nb * sizeof(unsigned long long) + (size_t)(nb + 2 * NB) * sizeof(int);
        if (smem > 48 * 1024) {
            cudaError_t e = cudaFuncSetAttribute(k_route_bucket, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            if (e != cudaSuccess) return e;
        }
        k_route_bucket<<<(unsigned)rows, kBucketThreads, smem, s>>>(scores, nb, NB, pval, k_floor, sorted, counts, hr);
        return cudaGetLastError();
    }
    // longer rows: CTA bitonic sort (E keys per thread)
    const int E = nbp / kCtaSortThreads;
    const size_t smem = (size_t)nbp * sizeof(unsigned long long);
    auto run = [&](auto kern) -> cudaError_t {
        if (smem > 48 * 1024) {
            cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            if (e != cudaSuccess) return e;
        }
        kern<<<(unsigned)rows, kCtaSortThreads, smem, s>>>(scores, nb, pval, k_floor, sorted, counts, hr);
        return cudaGetLastError();
    };
    switch (E) {
        case 2: return run(k_route_cta<2>);
        case 4: return run(k_route_cta<4>);
        case 8: return run(k_route_cta<8>);
        case 16: return run(k_route_cta<16>);
        default: return run(k_route_cta<32>);
    }
}

cudaError_t launch_route_stages(const bsa_plan& p, const void* q, const void* k, int dtype, double pval, int k_floor,
                                double* qbar, double* kbar, double* scores, uint16_t* sorted, int32_t* counts,
                                cudaStream_t s) {
    // one pass over all heads per stage (splitting heads into groups and running
    // pooling of one group beside the scores and sorts of another on a second
    // stream measured slower at 480p and 720p)
    cudaError_t e = launch_pool(p, q, k, dtype, qbar, kbar, s);
    if (e == cudaSuccess) e = launch_scores(p, qbar, kbar, scores, s);
    if (e == cudaSuccess) e = launch_route_rows(p, scores, pval, k_floor, sorted, counts, s);
    return e;
}

cudaError_t launch_scan_counts(const bsa_plan& p, const int32_t* counts, int32_t* row_ptr, float* L_h,
                               int64_t* nnz, int64_t col_cap, cudaStream_t s) {
    k_csr_scan<<<1, kScanThreads, 0, s>>>(counts, p.rows, (int)p.nb, row_ptr, L_h, nnz, col_cap, p.d_err);
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
