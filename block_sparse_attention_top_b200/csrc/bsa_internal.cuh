// Internal declarations shared by the libbsa translation units.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>
#include <stddef.h>

#include "bsa.h"

struct bsa_plan {
    int B, H, T, Hs, Ws, d, block, order;
    int64_t N, nb, rows;
    int device;
    int num_sms;
    int64_t l2_bytes;    // the device's L2 size (sizes the head groups of BSA_SCHED_L2_HEADS)
    int schedule;        // BSA_SCHED_*: order of the attention work list
    unsigned long long wait_ns;   // bound of the attention kernels' main-loop waits
    int32_t* d_perm;     // [N] raster index at reordered position
    int32_t* d_err;      // [4]: status, detail, spare, spare
};

namespace bsa {

constexpr size_t kAlign = 256;
constexpr int kMaxRouteBlocks = 8192;   // nb limit of the routing sort

inline size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// ---- route workspace layout (offsets in bytes) ----
struct RouteWs {
    size_t qbar, kbar, scores, sorted, counts, total;
};
RouteWs route_ws_layout(const bsa_plan& p);

// ---- attention workspace layout ----
// ---- mask workspace: per-row counts ----
inline size_t mask_ws_bytes(const bsa_plan& p) { return align_up((size_t)p.rows * sizeof(int32_t)); }
// BSA_OP_MASK: the counts plus, for the stripe producer, the block ranges
size_t stripe_ws_bytes(const bsa_plan& p);

struct AttnWs {
    size_t qp, kp, vp, work, hist, bins, counter, vscale, grank, total;
};
AttnWs attn_ws_layout(const bsa_plan& p);

// Device error recording: first status wins; detail holds an index.
__device__ __forceinline__ void record_error(int32_t* err, int status, int detail) {
    if (atomicCAS(err, 0, status) == 0) err[1] = detail;
}

// ---- launchers (return cudaError_t of the launch) ----
// The routing stages of bsa_route / bsa_route_static (pool, scores, row
// routing) into the given scratch on `s`; the CSR stage follows.
cudaError_t launch_route_stages(const bsa_plan& p, const void* q, const void* k, int dtype, double pval, int k_floor,
                                double* qbar, double* kbar, double* scores, uint16_t* sorted, int32_t* counts,
                                cudaStream_t s);
// Routing stages over heads h0 .. h0 + nh - 1 of every batch entry (nh <= 0:
// through the last head).
cudaError_t launch_pool(const bsa_plan& p, const void* q, const void* k, int dtype,
                        double* qbar, double* kbar, cudaStream_t s, int h0 = 0, int nh = 0);
cudaError_t launch_scores(const bsa_plan& p, const double* qbar, const double* kbar,
                          double* scores, cudaStream_t s, int h0 = 0, int nh = 0);
cudaError_t launch_route_rows(const bsa_plan& p, const double* scores, double pval, int k_floor,
                              uint16_t* sorted, int32_t* counts, cudaStream_t s, int h0 = 0, int nh = 0);
cudaError_t launch_csr(const bsa_plan& p, const int32_t* counts, const uint16_t* sorted,
                       int32_t* row_ptr, int32_t* col_idx, int64_t col_cap, float* L_h,
                       int64_t* nnz, cudaStream_t s);

// Exclusive scan of per-row counts -> row_ptr, nnz (and L_h unless null);
// BSA_ECAPACITY in the error word when nnz > col_cap.
cudaError_t launch_scan_counts(const bsa_plan& p, const int32_t* counts, int32_t* row_ptr, float* L_h,
                               int64_t* nnz, int64_t col_cap, cudaStream_t s);
cudaError_t launch_mask_window_anchor(const bsa_plan& p, int radius, int n_anchor, int step, int32_t* counts,
                                      int32_t* row_ptr, int32_t* col_idx, int64_t col_cap, int64_t* nnz,
                                      cudaStream_t s);
constexpr int kMaxMaskAnchors = 64;
// Stripe masks on the device: per-head parameters travel in the launch (at
// most kMaxStripeHeads heads); block frame/row ranges live in the workspace
// behind the per-row counts.
constexpr int kMaxStripeHeads = 160;
size_t stripe_ws_bytes(const bsa_plan& p);
cudaError_t launch_mask_stripes(const bsa_plan& p, const int32_t* params, int32_t* counts, void* ranges_ws,
                                int32_t* row_ptr, int32_t* col_idx, int64_t col_cap, int64_t* nnz, cudaStream_t s);
cudaError_t launch_augment(const bsa_plan& p, const int32_t* row_ptr, const uint16_t* order, const int32_t* extra,
                           int32_t* counts, int32_t* row_ptr_out, int32_t* col_idx_out, int64_t col_cap,
                           float* L_h_out, int64_t* nnz_out, cudaStream_t s);

// Work list in the plan's schedule.  hist and bins hold sched_bins(p) ints,
// grank B*H ints.
constexpr int kMaxSchedGroups = 8192;     // above: one group (heaviest-first)
int sched_heads_per_group(const bsa_plan& p);
int64_t sched_bins(const bsa_plan& p);
cudaError_t launch_worklist(const bsa_plan& p, const int32_t* row_ptr, int32_t* hist,
                            int32_t* bins, int32_t* grank, int32_t* work, cudaStream_t s);
// n_tensors = 3: Q, K and V; 2: Q and K only (V goes through launch_quant_v)
cudaError_t launch_permute(const bsa_plan& p, const void* q, const void* k, const void* v,
                           void* qp, void* kp, void* vp, cudaStream_t s, int n_tensors = 3);
cudaError_t launch_attn_simt(const bsa_plan& p, const void* qp, const void* kp, const void* vp,
                             const int32_t* row_ptr, const int32_t* col_idx, const int32_t* work,
                             void* o, cudaStream_t s);
cudaError_t launch_attn_tc(const bsa_plan& p, const void* qp, const void* kp, const void* vp,
                           const int32_t* row_ptr, const int32_t* col_idx, const int32_t* work,
                           int32_t* counter, void* o, cudaStream_t s);
// Ping-pong tensor-core kernel (two softmax warp groups on alternating key
// blocks); block = 128 only, d in {64, 128}.
bool attn_pp_supported(const bsa_plan& p);
// sigma != null: vp holds e4m3 V tiles from launch_quant_v and sigma their
// per-(head, channel) scales (the FP8 P.V product).
cudaError_t launch_attn_pp(const bsa_plan& p, const void* qp, const void* kp, const void* vp,
                           const int32_t* row_ptr, const int32_t* col_idx, const int32_t* work, void* o,
                           const float* sigma, cudaStream_t s);
// e4m3 V: sigma [B*H*d] floats (per head and channel), vt [B*H*nb*d, 128] bytes
cudaError_t launch_quant_v(const bsa_plan& p, const void* v, float* sigma, void* vt, cudaStream_t s);

// Host-side token order (no CUDA).
void token_order(int T, int Hs, int Ws, int order, int32_t* perm);

}  // namespace bsa
