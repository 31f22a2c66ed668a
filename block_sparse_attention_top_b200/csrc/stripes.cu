// Periodic diagonal stripe block masks, host and device producers (PSA pages: section 3.1,
// section 3.2 "Efficient and Flexible Kernel", appendix C.2 "Initialization
// of Mask Candidates" and appendix D "Locality-Induced Periodic Diagonal
// Stripes": per-head masks of an inter-frame and an intra-frame stripe
// family, each with a width, an offset and a stride, an infinite stride being
// a single diagonal, applied per block).  PSA's masks are searched offline
// per head and stay fixed, so a producer runs once per shape: on the host
// (bsa_mask_stripes) or on the device (bsa_mask_stripes_device, which writes
// the CSR straight into device memory); either CSR feeds bsa_sparse_attn like
// any other mask.
//
// Per head, params = (w_t, o_t, s_t, w_s, o_s, s_s): half-width, offset and
// stride over latent-frame offsets (inter-frame) and over row offsets inside
// a frame (intra-frame); stride <= 0 is infinite.  A family keeps key offset
// delta (key minus query) when |delta - o - n*s| <= w for some integer n.
// Blocks i (query) and j (key) of the token order are kept together when the
// inter-frame family keeps some frame offset between the two blocks' frame
// ranges and the intra-frame family some row offset between their row
// ranges ([min, max] over each block's tokens).  That holds when the offset
// interval [a, b] widened to [a - o - w, b - o + w] contains a multiple of s
// (contains 0 for an infinite stride).
//
// Device producer, for a plan: k_stripe_ranges takes each block's frame and
// row range through the plan's token order; k_stripe_rows counts each row's
// kept blocks (one warp per row, 32 key blocks per step), the routing CSR
// scan turns the counts into row_ptr and nnz, and k_stripe_rows writes the
// ascending columns (a ballot prefix orders each step's columns).
#include <algorithm>
#include <vector>

#include "bsa_internal.cuh"

namespace {

__host__ __device__ inline int64_t floor_div(int64_t a, int64_t d) {
    return a >= 0 ? a / d : -((-a + d - 1) / d);
}

__host__ __device__ inline bool family_keeps(int64_t a, int64_t b, int w, int o, int s) {
    const int64_t lo = a - o - w, hi = b - o + w;
    if (s <= 0) return lo <= 0 && 0 <= hi;
    return floor_div(hi, s) * s >= lo;
}

struct StripeParams {
    int32_t v[6 * bsa::kMaxStripeHeads];
};

// ranges[i] = (first frame, last frame, first row, last row) of block i's tokens
__global__ void k_stripe_ranges(const int32_t* __restrict__ perm, int N, int block, int Ws, int hw, int nb,
                                int4* __restrict__ ranges) {
    const int i = blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    if (i >= nb) return;
    int f_lo = INT32_MAX, f_hi = INT32_MIN, y_lo = INT32_MAX, y_hi = INT32_MIN;
    for (int n = i * block + lane; n < min(N, (i + 1) * block); n += 32) {
        const int tok = perm[n], t = tok / hw, y = (tok % hw) / Ws;
        f_lo = min(f_lo, t); f_hi = max(f_hi, t);
        y_lo = min(y_lo, y); y_hi = max(y_hi, y);
    }
    for (int o = 16; o > 0; o >>= 1) {
        f_lo = min(f_lo, __shfl_xor_sync(0xffffffffu, f_lo, o));
        f_hi = max(f_hi, __shfl_xor_sync(0xffffffffu, f_hi, o));
        y_lo = min(y_lo, __shfl_xor_sync(0xffffffffu, y_lo, o));
        y_hi = max(y_hi, __shfl_xor_sync(0xffffffffu, y_hi, o));
    }
    if (lane == 0) ranges[i] = make_int4(f_lo, f_hi, y_lo, y_hi);
}

// FILL = false: counts[r] = kept blocks of row r; FILL = true: write them at row_ptr[r].
template <bool FILL>
__global__ void k_stripe_rows(const __grid_constant__ StripeParams prm, const int4* __restrict__ ranges,
                              int64_t rows, int H, int nb, int32_t* __restrict__ counts,
                              const int32_t* __restrict__ row_ptr, int32_t* __restrict__ col_idx, int64_t col_cap) {
    const int64_t r = (int64_t)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    if (r >= rows) return;
    const int i = (int)(r % nb), h = (int)((r / nb) % H);
    const int32_t* pr = prm.v + 6 * h;
    const int4 qi = ranges[i];
    int64_t pos = FILL ? row_ptr[r] : 0;
    int total = 0;
    for (int j0 = 0; j0 < nb; j0 += 32) {
        const int j = j0 + lane;
        bool keep = false;
        if (j < nb) {
            const int4 kj = ranges[j];
            keep = family_keeps((int64_t)kj.x - qi.y, (int64_t)kj.y - qi.x, pr[0], pr[1], pr[2]) &&
                   family_keeps((int64_t)kj.z - qi.w, (int64_t)kj.w - qi.z, pr[3], pr[4], pr[5]);
        }
        const unsigned ballot = __ballot_sync(0xffffffffu, keep);
        if (FILL && keep) {
            const int64_t at = pos + __popc(ballot & ((1u << lane) - 1u));
            if (at < col_cap) col_idx[at] = j;
        }
        pos += __popc(ballot);
        total += __popc(ballot);
    }
    if (!FILL && lane == 0) counts[r] = total;
}

}  // namespace

namespace bsa {

size_t stripe_ws_bytes(const bsa_plan& p) { return align_up((size_t)p.nb * sizeof(int4)); }

cudaError_t launch_mask_stripes(const bsa_plan& p, const int32_t* params, int32_t* counts, void* ranges_ws,
                                int32_t* row_ptr, int32_t* col_idx, int64_t col_cap, int64_t* nnz, cudaStream_t s) {
    StripeParams sp{};
    for (int e = 0; e < 6 * p.H; ++e) sp.v[e] = params[e];
    int4* ranges = (int4*)ranges_ws;
    const int t = 256, wpb = t / 32;
    k_stripe_ranges<<<(unsigned)((p.nb + wpb - 1) / wpb), t, 0, s>>>(p.d_perm, (int)p.N, p.block, p.Ws,
                                                                     p.Hs * p.Ws, (int)p.nb, ranges);
    const unsigned g = (unsigned)((p.rows + wpb - 1) / wpb);
    k_stripe_rows<false><<<g, t, 0, s>>>(sp, ranges, p.rows, p.H, (int)p.nb, counts, nullptr, nullptr, 0);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    e = launch_scan_counts(p, counts, row_ptr, nullptr, nnz, col_cap, s);
    if (e != cudaSuccess) return e;
    if (col_cap == 0) return cudaSuccess;
    k_stripe_rows<true><<<g, t, 0, s>>>(sp, ranges, p.rows, p.H, (int)p.nb, nullptr, row_ptr, col_idx, col_cap);
    return cudaGetLastError();
}

}  // namespace bsa

extern "C" int bsa_mask_stripes(int B, int H, int T, int Hs, int Ws, int block, int order, const int32_t* params,
                                int32_t* row_ptr, int32_t* col_idx, int64_t col_cap, int64_t* nnz) {
    if (B < 1 || H < 1 || T < 1 || Hs < 1 || Ws < 1 || (block != 64 && block != 128)) return BSA_EINVAL;
    if (order != BSA_ORDER_HILBERT2D_FRAME && order != BSA_ORDER_IDENTITY) return BSA_EINVAL;
    if (!params || !row_ptr || !nnz || col_cap < 0 || (col_cap > 0 && !col_idx)) return BSA_EINVAL;
    for (int h = 0; h < H; ++h)
        if (params[6 * h + 0] < 0 || params[6 * h + 3] < 0) return BSA_EINVAL;   // widths
    const int64_t N = (int64_t)T * Hs * Ws;
    if (N > INT32_MAX) return BSA_EUNSUPPORTED;
    const int64_t nb = (N + block - 1) / block;
    const int64_t rows = (int64_t)B * H * nb;
    if (rows * nb > INT32_MAX) return BSA_EUNSUPPORTED;       // row_ptr values are int32

    std::vector<int32_t> perm((size_t)N);
    bsa::token_order(T, Hs, Ws, order, perm.data());
    const int64_t hw = (int64_t)Hs * Ws;
    std::vector<int64_t> f_lo(nb), f_hi(nb), y_lo(nb), y_hi(nb);
    for (int64_t i = 0; i < nb; ++i) {
        f_lo[i] = y_lo[i] = INT64_MAX;
        f_hi[i] = y_hi[i] = INT64_MIN;
        for (int64_t n = i * block; n < std::min(N, (i + 1) * block); ++n) {
            const int64_t t = perm[n] / hw, y = (perm[n] % hw) / Ws;
            f_lo[i] = std::min(f_lo[i], t);
            f_hi[i] = std::max(f_hi[i], t);
            y_lo[i] = std::min(y_lo[i], y);
            y_hi[i] = std::max(y_hi[i], y);
        }
    }
    // the kept columns of every head's query blocks, then the CSR over (b, h, i)
    std::vector<std::vector<int32_t>> cols((size_t)(H * nb));
    for (int h = 0; h < H; ++h) {
        const int32_t* pr = params + 6 * h;
        for (int64_t i = 0; i < nb; ++i) {
            std::vector<int32_t>& c = cols[(size_t)(h * nb + i)];
            for (int64_t j = 0; j < nb; ++j)
                if (family_keeps(f_lo[j] - f_hi[i], f_hi[j] - f_lo[i], pr[0], pr[1], pr[2]) &&
                    family_keeps(y_lo[j] - y_hi[i], y_hi[j] - y_lo[i], pr[3], pr[4], pr[5]))
                    c.push_back((int32_t)j);
        }
    }
    int64_t total = 0;
    row_ptr[0] = 0;
    int64_t r = 0;
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h)
            for (int64_t i = 0; i < nb; ++i, ++r) {
                for (int32_t j : cols[(size_t)(h * nb + i)]) {
                    if (total < col_cap) col_idx[total] = j;
                    ++total;
                }
                row_ptr[r + 1] = (int32_t)total;
            }
    *nnz = total;
    return total > col_cap ? BSA_ECAPACITY : BSA_OK;
}
