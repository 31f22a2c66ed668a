// Periodic diagonal stripe block masks, host producer (PSA pages: section 3.1,
// section 3.2 "Efficient and Flexible Kernel", appendix C.2 "Initialization
// of Mask Candidates" and appendix D "Locality-Induced Periodic Diagonal
// Stripes": per-head masks of an inter-frame and an intra-frame stripe
// family, each with a width, an offset and a stride, an infinite stride being
// a single diagonal, applied per block).  PSA's masks are searched offline
// per head and stay fixed, so the producer runs once per shape on the host;
// the CSR it writes feeds bsa_sparse_attn like any other mask.
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
#include <algorithm>
#include <vector>

#include "bsa_internal.cuh"

namespace {

int64_t floor_div(int64_t a, int64_t d) { return a >= 0 ? a / d : -((-a + d - 1) / d); }

bool family_keeps(int64_t a, int64_t b, int w, int o, int s) {
    const int64_t lo = a - o - w, hi = b - o + w;
    if (s <= 0) return lo <= 0 && 0 <= hi;
    return floor_div(hi, s) * s >= lo;
}

}  // namespace

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
