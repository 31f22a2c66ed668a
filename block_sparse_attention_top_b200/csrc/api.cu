// libbsa C ABI: plans, argument validation, workspace layout, stream-ordered
// launch sequences.  Kernels live in route.cu, route_static.cu, masks.cu,
// augment.cu, prepare.cu, attn_pp.cu (block 128), attn_tc.cu (block 64) and
// attn_simt.cu; balance.cu is host code.
#include <algorithm>
#include <cmath>
#include <cstring>
#include <new>
#include <vector>

#include "bsa_internal.cuh"

namespace bsa {

// Hilbert index of cell (x, y) on a 2^m x 2^m curve (the classic 2-D curve:
// quadrants visited lower-left, upper-left, upper-right, lower-right, with the
// lower quadrants' sub-curves transposed, the lower-right one also reflected).
// Walks the bit planes from the top; after reading a plane the remaining
// low bits are mapped into the frame of that quadrant's sub-curve.
static uint64_t hilbert_index(uint32_t side, uint32_t x, uint32_t y) {
    uint64_t d = 0;
    for (uint32_t s = side >> 1; s > 0; s >>= 1) {
        const uint32_t rx = (x & s) ? 1u : 0u;
        const uint32_t ry = (y & s) ? 1u : 0u;
        // quadrant rank along the curve: (rx,ry) = (0,0)->0, (0,1)->1, (1,1)->2, (1,0)->3
        d += (uint64_t)s * s * ((3u * rx) ^ ry);
        x &= s - 1;
        y &= s - 1;
        if (ry == 0) {
            if (rx == 1) { x = s - 1 - x; y = s - 1 - y; }
            const uint32_t t = x; x = y; y = t;
        }
    }
    return d;
}

void token_order(int T, int Hs, int Ws, int order, int32_t* perm) {
    const int64_t hw = (int64_t)Hs * Ws;
    if (order == BSA_ORDER_IDENTITY) {
        for (int64_t n = 0; n < (int64_t)T * hw; ++n) perm[n] = (int32_t)n;
        return;
    }
    uint32_t side = 1;
    while (side < (uint32_t)std::max(Hs, Ws)) side <<= 1;
    std::vector<std::pair<uint64_t, int32_t>> cells((size_t)hw);
    for (int y = 0; y < Hs; ++y)
        for (int x = 0; x < Ws; ++x)
            cells[(size_t)y * Ws + x] = {hilbert_index(side, (uint32_t)x, (uint32_t)y), (int32_t)(y * Ws + x)};
    std::sort(cells.begin(), cells.end());
    for (int t = 0; t < T; ++t)
        for (int64_t c = 0; c < hw; ++c) perm[t * hw + c] = (int32_t)(t * hw + cells[(size_t)c].second);
}

RouteWs route_ws_layout(const bsa_plan& p) {
    RouteWs w{};
    size_t off = 0;
    const size_t pooled = (size_t)p.rows * p.d * sizeof(double);
    w.qbar = off;   off += align_up(pooled);
    w.kbar = off;   off += align_up(pooled);
    w.scores = off; off += align_up((size_t)p.rows * p.nb * sizeof(double));
    w.sorted = off; off += align_up((size_t)p.rows * p.nb * sizeof(uint16_t));
    w.counts = off; off += align_up((size_t)p.rows * sizeof(int32_t));
    w.total = off;
    return w;
}

AttnWs attn_ws_layout(const bsa_plan& p) {
    AttnWs w{};
    size_t off = 0;
    const size_t tile = (size_t)p.B * p.H * p.nb * p.block * p.d * 2;   // bf16
    w.qp = off; off += align_up(tile);
    w.kp = off; off += align_up(tile);
    w.vp = off; off += align_up(tile);
    w.work = off; off += align_up((size_t)p.rows * sizeof(int32_t));
    w.hist = off; off += align_up((size_t)sched_bins(p) * sizeof(int32_t));
    w.bins = off; off += align_up((size_t)sched_bins(p) * sizeof(int32_t));
    w.counter = off; off += align_up(4 * sizeof(int32_t));
    w.vscale = off; off += align_up((size_t)p.B * p.H * p.d * sizeof(float));   // e4m3 V: per-channel scales
    w.grank = off; off += align_up((size_t)p.B * p.H * sizeof(int32_t));       // head-group ranks
    w.total = off;
    return w;
}

}  // namespace bsa

using namespace bsa;

static bool misaligned(const void* ptr, size_t a) { return ((uintptr_t)ptr) % a != 0; }

extern "C" {

const char* bsa_strerror(int status) {
    switch (status) {
        case BSA_OK: return "ok";
        case BSA_EINVAL: return "invalid argument";
        case BSA_EUNSUPPORTED: return "unsupported shape or device";
        case BSA_ECAPACITY: return "routed nnz exceeded col_cap";
        case BSA_EWORKSPACE: return "workspace missing, too small or misaligned";
        case BSA_ECUDA: return "CUDA runtime error";
        case BSA_EDEVICE: return "device-side check failed (malformed mask or expired wait)";
        default: return "unknown status";
    }
}

int bsa_token_order(int T, int Hs, int Ws, int order, int32_t* perm) {
    if (!perm || T < 1 || Hs < 1 || Ws < 1) return BSA_EINVAL;
    if (order != BSA_ORDER_HILBERT2D_FRAME && order != BSA_ORDER_IDENTITY) return BSA_EINVAL;
    if ((int64_t)T * Hs * Ws > INT32_MAX) return BSA_EUNSUPPORTED;
    token_order(T, Hs, Ws, order, perm);
    return BSA_OK;
}

int bsa_plan_create(bsa_plan** out, int B, int H, int T, int Hs, int Ws,
                    int head_dim, int block, int order) {
    if (!out) return BSA_EINVAL;
    *out = nullptr;
    if (B < 1 || H < 1 || T < 1 || Hs < 1 || Ws < 1) return BSA_EINVAL;
    if (order != BSA_ORDER_HILBERT2D_FRAME && order != BSA_ORDER_IDENTITY) return BSA_EINVAL;
    if (head_dim != 64 && head_dim != 128) return BSA_EUNSUPPORTED;
    if (block != 64 && block != 128) return BSA_EUNSUPPORTED;
    const int64_t N = (int64_t)T * Hs * Ws;
    const int64_t nb = (N + block - 1) / block;
    // element indices of [B,N,H,d] and of the padded tiles must fit in int64 and
    // row indices in int32
    if (N > (1ll << 30) || (int64_t)B * H * nb > (1ll << 30)) return BSA_EUNSUPPORTED;
    // the attention kernels address the padded tiles with 32-bit row coordinates
    if ((int64_t)B * H * nb * block > INT32_MAX) return BSA_EUNSUPPORTED;

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return BSA_ECUDA;
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return BSA_ECUDA;
    if (prop.major != 10 || prop.minor != 0) return BSA_EUNSUPPORTED;

    bsa_plan* p = new (std::nothrow) bsa_plan();
    if (!p) return BSA_ECUDA;
    p->B = B; p->H = H; p->T = T; p->Hs = Hs; p->Ws = Ws; p->d = head_dim; p->block = block;
    p->order = order; p->N = N; p->nb = nb; p->rows = (int64_t)B * H * nb;
    p->device = dev; p->num_sms = prop.multiProcessorCount;
    p->l2_bytes = prop.l2CacheSize; p->schedule = BSA_SCHED_L2_HEADS;
    p->wait_ns = 4000000000ull;
    std::vector<int32_t> perm((size_t)N);
    token_order(T, Hs, Ws, order, perm.data());
    const bool ok = cudaMalloc(&p->d_perm, (size_t)N * sizeof(int32_t)) == cudaSuccess &&
                    cudaMalloc(&p->d_err, 4 * sizeof(int32_t)) == cudaSuccess &&
                    cudaMemcpy(p->d_perm, perm.data(), (size_t)N * sizeof(int32_t), cudaMemcpyHostToDevice) ==
                        cudaSuccess &&
                    cudaMemset(p->d_err, 0, 4 * sizeof(int32_t)) == cudaSuccess;
    if (!ok) {
        bsa_plan_destroy(p);
        return BSA_ECUDA;
    }
    *out = p;
    return BSA_OK;
}

void bsa_plan_destroy(bsa_plan* p) {
    if (!p) return;
    cudaFree(p->d_perm);
    cudaFree(p->d_err);
    delete p;
}

int bsa_plan_info(const bsa_plan* p, int64_t* N, int64_t* nb, int64_t* rows) {
    if (!p) return BSA_EINVAL;
    if (N) *N = p->N;
    if (nb) *nb = p->nb;
    if (rows) *rows = p->rows;
    return BSA_OK;
}

int bsa_plan_set_schedule(bsa_plan* p, int schedule) {
    if (!p) return BSA_EINVAL;
    if (schedule != BSA_SCHED_L2_HEADS && schedule != BSA_SCHED_HEAVIEST_FIRST && schedule != BSA_SCHED_IN_ORDER)
        return BSA_EINVAL;
    p->schedule = schedule;
    return BSA_OK;
}

int bsa_plan_set_wait_limit(bsa_plan* p, uint64_t ns) {
    if (!p) return BSA_EINVAL;
    p->wait_ns = ns;
    return BSA_OK;
}

int bsa_schedule_balance(const bsa_plan* p, const int32_t* row_ptr, const int32_t* work, double* rho,
                         int64_t* max_blocks, double* mean_blocks) {
    if (!p || !row_ptr || !work || !rho) return BSA_EINVAL;
    // the attention kernels' static assignment: one CTA per SM, item k*grid + c
    // to CTA c on even rounds k and to CTA grid - 1 - c on odd rounds
    const int64_t grid = std::min<int64_t>(p->num_sms, p->rows);
    std::vector<int64_t> load((size_t)grid, 0);
    for (int64_t idx = 0; idx < p->rows; ++idx) {
        const int64_t k = idx / grid, c = idx % grid;
        const int64_t cta = (k & 1) ? grid - 1 - c : c;
        const int32_t r = work[idx];
        if (r < 0 || r >= p->rows) return BSA_EINVAL;
        const int64_t n = (int64_t)row_ptr[r + 1] - row_ptr[r];
        if (n < 0 || n > p->nb) return BSA_EINVAL;
        load[(size_t)cta] += n;
    }
    int64_t mx = 0, sum = 0;
    for (int64_t v : load) { mx = std::max(mx, v); sum += v; }
    const double mean = grid > 0 ? (double)sum / (double)grid : 0.0;
    *rho = mean > 0 ? (double)mx / mean : 1.0;
    if (max_blocks) *max_blocks = mx;
    if (mean_blocks) *mean_blocks = mean;
    return BSA_OK;
}

int bsa_attn_intermediates(const bsa_plan* p, void* ws, const int32_t** work, const void** v_e4m3,
                           const float** v_scale) {
    if (!p || !ws) return BSA_EINVAL;
    const AttnWs L = attn_ws_layout(*p);
    char* base = (char*)ws;
    if (work) *work = (const int32_t*)(base + L.work);
    if (v_e4m3) *v_e4m3 = (const void*)(base + L.vp);
    if (v_scale) *v_scale = (const float*)(base + L.vscale);
    return BSA_OK;
}

size_t bsa_workspace_size(const bsa_plan* p, int op) {
    if (!p) return 0;
    if (op == BSA_OP_ROUTE) return route_ws_layout(*p).total;
    if (op == BSA_OP_ATTN) return attn_ws_layout(*p).total;
    if (op == BSA_OP_MASK) return mask_ws_bytes(*p) + stripe_ws_bytes(*p);
    if (op == BSA_OP_AUGMENT) return mask_ws_bytes(*p);
    return 0;
}

static int check_ws(void* ws, size_t ws_bytes, size_t need) {
    if (!ws || misaligned(ws, kAlign) || ws_bytes < need) return BSA_EWORKSPACE;
    return BSA_OK;
}

#define BSA_LAUNCH(call) do { if ((call) != cudaSuccess) return BSA_ECUDA; } while (0)

int bsa_route(const bsa_plan* p, const void* q, const void* k, int dtype, float pval, int k_floor,
              int32_t* row_ptr, int32_t* col_idx, int64_t col_cap, float* L_h, int64_t* nnz,
              void* ws, size_t ws_bytes, void* stream) {
    if (!p || !q || !k || !row_ptr || !L_h || !nnz) return BSA_EINVAL;
    if (col_cap < 0 || (col_cap > 0 && !col_idx)) return BSA_EINVAL;
    if (dtype != BSA_BF16 && dtype != BSA_F32) return BSA_EINVAL;
    if (!(pval > 0.0f) || !(pval <= 1.0f) || k_floor < 0) return BSA_EINVAL;
    if (misaligned(q, 16) || misaligned(k, 16) || misaligned(row_ptr, 4) ||
        (col_idx && misaligned(col_idx, 4)) || misaligned(L_h, 4) || misaligned(nnz, 8))
        return BSA_EINVAL;
    if (p->nb > kMaxRouteBlocks) return BSA_EUNSUPPORTED;
    if (p->rows * p->nb > INT32_MAX) return BSA_EUNSUPPORTED;    // worst-case nnz must fit row_ptr (int32)
    const RouteWs L = route_ws_layout(*p);
    if (int rc = check_ws(ws, ws_bytes, L.total)) return rc;
    cudaStream_t s = (cudaStream_t)stream;
    char* base = (char*)ws;
    double* qbar = (double*)(base + L.qbar);
    double* kbar = (double*)(base + L.kbar);
    double* scores = (double*)(base + L.scores);
    uint16_t* sorted = (uint16_t*)(base + L.sorted);
    int32_t* counts = (int32_t*)(base + L.counts);
    BSA_LAUNCH(launch_route_stages(*p, q, k, dtype, (double)pval, k_floor, qbar, kbar, scores, sorted, counts, s));
    BSA_LAUNCH(launch_csr(*p, counts, sorted, row_ptr, col_idx, col_cap, L_h, nnz, s));
    return BSA_OK;
}

int bsa_route_order(const bsa_plan* p, void* ws, const uint16_t** order) {
    if (!p || !ws || !order) return BSA_EINVAL;
    *order = (const uint16_t*)((char*)ws + route_ws_layout(*p).sorted);
    return BSA_OK;
}

int bsa_augment(const bsa_plan* p, const int32_t* row_ptr, const uint16_t* order, const int32_t* extra,
                int32_t* row_ptr_out, int32_t* col_idx_out, int64_t col_cap, float* L_h_out, int64_t* nnz_out,
                void* ws, size_t ws_bytes, void* stream) {
    if (!p || !row_ptr || !order || !extra || !row_ptr_out || !L_h_out || !nnz_out) return BSA_EINVAL;
    if (col_cap < 0 || (col_cap > 0 && !col_idx_out)) return BSA_EINVAL;
    if (misaligned(row_ptr, 4) || misaligned(order, 2) || misaligned(extra, 4) || misaligned(row_ptr_out, 4) ||
        (col_idx_out && misaligned(col_idx_out, 4)) || misaligned(L_h_out, 4) || misaligned(nnz_out, 8))
        return BSA_EINVAL;
    if (p->rows * p->nb > INT32_MAX) return BSA_EUNSUPPORTED;    // worst-case nnz must fit row_ptr (int32)
    if (int rc = check_ws(ws, ws_bytes, mask_ws_bytes(*p))) return rc;
    BSA_LAUNCH(launch_augment(*p, row_ptr, order, extra, (int32_t*)ws, row_ptr_out, col_idx_out, col_cap, L_h_out,
                              nnz_out, (cudaStream_t)stream));
    return BSA_OK;
}

int bsa_sasa_budget(int R, const float* L_r, float n1, float n2, float S, float* B_r, float* L_aug, float* A,
                    const int32_t* heads_per_rank, int32_t* extra_per_head) {
    if (R < 1 || !L_r || !B_r) return BSA_EINVAL;
    if (heads_per_rank && !extra_per_head) return BSA_EINVAL;
    double lmax = L_r[0];
    for (int r = 1; r < R; ++r) lmax = std::max(lmax, (double)L_r[r]);
    double amax = -1e300;
    int64_t h = 0;
    for (int r = 0; r < R; ++r) {
        const double dl = lmax - (double)L_r[r];
        const double b = dl > (double)n2 * lmax ? (double)n1 * dl : 0.0;
        B_r[r] = (float)b;
        const double la = (double)L_r[r] + b;
        if (L_aug) L_aug[r] = (float)la;
        amax = std::max(amax, la);
        if (heads_per_rank) {
            if (heads_per_rank[r] < 1) return BSA_EINVAL;
            const int32_t e = (int32_t)std::floor(b / heads_per_rank[r]);
            for (int32_t t = 0; t < heads_per_rank[r]; ++t) extra_per_head[h++] = e;
        }
    }
    if (A) *A = (float)(std::max(0.0, amax - lmax) + (double)S);
    return BSA_OK;
}

int bsa_mask_window_anchor(const bsa_plan* p, int radius_frames, int n_anchor, int step, int32_t* row_ptr,
                           int32_t* col_idx, int64_t col_cap, int64_t* nnz, void* ws, size_t ws_bytes,
                           void* stream) {
    if (!p || !row_ptr || !nnz || radius_frames < 0 || n_anchor < 0 || n_anchor > kMaxMaskAnchors || step < 0)
        return BSA_EINVAL;
    if (col_cap < 0 || (col_cap > 0 && !col_idx)) return BSA_EINVAL;
    if (misaligned(row_ptr, 4) || (col_idx && misaligned(col_idx, 4)) || misaligned(nnz, 8)) return BSA_EINVAL;
    if (p->rows * p->nb > INT32_MAX) return BSA_EUNSUPPORTED;    // worst-case nnz must fit row_ptr (int32)
    if (int rc = check_ws(ws, ws_bytes, mask_ws_bytes(*p))) return rc;
    BSA_LAUNCH(launch_mask_window_anchor(*p, radius_frames, n_anchor, step, (int32_t*)ws, row_ptr, col_idx, col_cap,
                                         nnz, (cudaStream_t)stream));
    return BSA_OK;
}

int bsa_mask_stripes_device(const bsa_plan* p, const int32_t* params, int32_t* row_ptr, int32_t* col_idx,
                            int64_t col_cap, int64_t* nnz, void* ws, size_t ws_bytes, void* stream) {
    if (!p || !params || !row_ptr || !nnz) return BSA_EINVAL;
    if (col_cap < 0 || (col_cap > 0 && !col_idx)) return BSA_EINVAL;
    if (misaligned(row_ptr, 4) || (col_idx && misaligned(col_idx, 4)) || misaligned(nnz, 8)) return BSA_EINVAL;
    for (int h = 0; h < p->H; ++h)
        if (params[6 * h + 0] < 0 || params[6 * h + 3] < 0) return BSA_EINVAL;   // widths
    if (p->H > kMaxStripeHeads) return BSA_EUNSUPPORTED;
    if (p->rows * p->nb > INT32_MAX) return BSA_EUNSUPPORTED;    // worst-case nnz must fit row_ptr (int32)
    const size_t counts_bytes = mask_ws_bytes(*p);
    if (int rc = check_ws(ws, ws_bytes, counts_bytes + stripe_ws_bytes(*p))) return rc;
    BSA_LAUNCH(launch_mask_stripes(*p, params, (int32_t*)ws, (char*)ws + counts_bytes, row_ptr, col_idx, col_cap,
                                   nnz, (cudaStream_t)stream));
    return BSA_OK;
}

int bsa_route_intermediates(const bsa_plan* p, void* ws, const double** qbar,
                            const double** kbar, const double** scores) {
    if (!p || !ws) return BSA_EINVAL;
    const RouteWs L = route_ws_layout(*p);
    char* base = (char*)ws;
    if (qbar) *qbar = (const double*)(base + L.qbar);
    if (kbar) *kbar = (const double*)(base + L.kbar);
    if (scores) *scores = (const double*)(base + L.scores);
    return BSA_OK;
}

int bsa_attn_prepare(const bsa_plan* p, const void* q, const void* k, const void* v,
                     const int32_t* row_ptr, void* ws, size_t ws_bytes, void* stream) {
    if (!p || !q || !k || !v || !row_ptr) return BSA_EINVAL;
    if (misaligned(q, 16) || misaligned(k, 16) || misaligned(v, 16) || misaligned(row_ptr, 4))
        return BSA_EINVAL;
    const AttnWs L = attn_ws_layout(*p);
    if (int rc = check_ws(ws, ws_bytes, L.total)) return rc;
    cudaStream_t s = (cudaStream_t)stream;
    char* base = (char*)ws;
    BSA_LAUNCH(launch_worklist(*p, row_ptr, (int32_t*)(base + L.hist), (int32_t*)(base + L.bins),
                               (int32_t*)(base + L.grank), (int32_t*)(base + L.work), s));
    BSA_LAUNCH(launch_permute(*p, q, k, v, base + L.qp, base + L.kp, base + L.vp, s));
    return BSA_OK;
}

static int attn_run_common(const bsa_plan* p, const int32_t* row_ptr, const int32_t* col_idx,
                           void* o, void* ws, size_t ws_bytes, void* stream, bool simt) {
    if (!p || !row_ptr || !col_idx || !o) return BSA_EINVAL;
    if (misaligned(o, 16) || misaligned(row_ptr, 4) || misaligned(col_idx, 4)) return BSA_EINVAL;
    const AttnWs L = attn_ws_layout(*p);
    if (int rc = check_ws(ws, ws_bytes, L.total)) return rc;
    cudaStream_t s = (cudaStream_t)stream;
    char* base = (char*)ws;
    if (simt) {
        BSA_LAUNCH(launch_attn_simt(*p, base + L.qp, base + L.kp, base + L.vp, row_ptr, col_idx,
                                    (const int32_t*)(base + L.work), o, s));
    } else if (attn_pp_supported(*p)) {
        BSA_LAUNCH(launch_attn_pp(*p, base + L.qp, base + L.kp, base + L.vp, row_ptr, col_idx,
                                  (const int32_t*)(base + L.work), o, nullptr, s));
    } else {
        BSA_LAUNCH(launch_attn_tc(*p, base + L.qp, base + L.kp, base + L.vp, row_ptr, col_idx,
                                  (const int32_t*)(base + L.work), (int32_t*)(base + L.counter), o, s));
    }
    return BSA_OK;
}

int bsa_attn_run(const bsa_plan* p, const int32_t* row_ptr, const int32_t* col_idx, void* o,
                 void* ws, size_t ws_bytes, void* stream) {
    return attn_run_common(p, row_ptr, col_idx, o, ws, ws_bytes, stream, false);
}

int bsa_attn_run_simt(const bsa_plan* p, const int32_t* row_ptr, const int32_t* col_idx, void* o,
                      void* ws, size_t ws_bytes, void* stream) {
    return attn_run_common(p, row_ptr, col_idx, o, ws, ws_bytes, stream, true);
}

int bsa_sparse_attn(const bsa_plan* p, const void* q, const void* k, const void* v,
                    const int32_t* row_ptr, const int32_t* col_idx, void* o,
                    void* ws, size_t ws_bytes, void* stream) {
    if (!col_idx || !o) return BSA_EINVAL;
    if (int rc = bsa_attn_prepare(p, q, k, v, row_ptr, ws, ws_bytes, stream)) return rc;
    return bsa_attn_run(p, row_ptr, col_idx, o, ws, ws_bytes, stream);
}

// ---- FP8 (e4m3) P.V product ----
int bsa_attn_prepare_fp8v(const bsa_plan* p, const void* q, const void* k, const void* v,
                          const int32_t* row_ptr, void* ws, size_t ws_bytes, void* stream) {
    if (!p || !q || !k || !v || !row_ptr) return BSA_EINVAL;
    if (misaligned(q, 16) || misaligned(k, 16) || misaligned(v, 16) || misaligned(row_ptr, 4))
        return BSA_EINVAL;
    if (!attn_pp_supported(*p)) return BSA_EUNSUPPORTED;
    const AttnWs L = attn_ws_layout(*p);
    if (int rc = check_ws(ws, ws_bytes, L.total)) return rc;
    cudaStream_t s = (cudaStream_t)stream;
    char* base = (char*)ws;
    BSA_LAUNCH(launch_worklist(*p, row_ptr, (int32_t*)(base + L.hist), (int32_t*)(base + L.bins),
                               (int32_t*)(base + L.grank), (int32_t*)(base + L.work), s));
    BSA_LAUNCH(launch_permute(*p, q, k, v, base + L.qp, base + L.kp, nullptr, s, 2));
    BSA_LAUNCH(launch_quant_v(*p, v, (float*)(base + L.vscale), base + L.vp, s));
    return BSA_OK;
}

int bsa_attn_run_fp8v(const bsa_plan* p, const int32_t* row_ptr, const int32_t* col_idx, void* o,
                      void* ws, size_t ws_bytes, void* stream) {
    if (!p || !row_ptr || !col_idx || !o) return BSA_EINVAL;
    if (misaligned(o, 16) || misaligned(row_ptr, 4) || misaligned(col_idx, 4)) return BSA_EINVAL;
    if (!attn_pp_supported(*p)) return BSA_EUNSUPPORTED;
    const AttnWs L = attn_ws_layout(*p);
    if (int rc = check_ws(ws, ws_bytes, L.total)) return rc;
    char* base = (char*)ws;
    BSA_LAUNCH(launch_attn_pp(*p, base + L.qp, base + L.kp, base + L.vp, row_ptr, col_idx,
                              (const int32_t*)(base + L.work), o, (const float*)(base + L.vscale),
                              (cudaStream_t)stream));
    return BSA_OK;
}

int bsa_sparse_attn_fp8v(const bsa_plan* p, const void* q, const void* k, const void* v,
                         const int32_t* row_ptr, const int32_t* col_idx, void* o,
                         void* ws, size_t ws_bytes, void* stream) {
    if (!col_idx || !o) return BSA_EINVAL;
    if (int rc = bsa_attn_prepare_fp8v(p, q, k, v, row_ptr, ws, ws_bytes, stream)) return rc;
    return bsa_attn_run_fp8v(p, row_ptr, col_idx, o, ws, ws_bytes, stream);
}

int bsa_last_device_error(const bsa_plan* p, void* stream) {
    if (!p) return BSA_EINVAL;
    cudaStream_t s = (cudaStream_t)stream;
    if (cudaStreamSynchronize(s) != cudaSuccess) return BSA_ECUDA;
    int32_t h[4] = {0, 0, 0, 0};
    if (cudaMemcpy(h, p->d_err, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess) return BSA_ECUDA;
    if (cudaMemset(p->d_err, 0, sizeof(h)) != cudaSuccess) return BSA_ECUDA;
    return h[0];
}

}  // extern "C"
