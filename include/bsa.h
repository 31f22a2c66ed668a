/*
 * bsa.h -- C ABI of libbsa: Top-p block routing and block-sparse attention
 * for video diffusion transformers, hand-written for B200 (sm_100a).
 *
 * What it computes follows the FVAttn pages:
 *   - routing: FVAttn review, section 3 "Stage 1: Sparse Mask Routing" and
 *     section 3.1 "Sparse Routing Frontend" (Hilbert block reordering, Top-p
 *     CDF threshold, Top-k safety floor, per-head workload and key-block
 *     importance order); alanhou.org blog, "Key Concepts" (the minimum number
 *     of blocks whose cumulative attention weight reaches p, and at least k
 *     blocks); the workload L_h is the review's Eq. 1;
 *   - attention: FVAttn review, section 3 "Block-Sparse Attention Execution"
 *     (attention over the retained blocks, then head-order / token-order
 *     restoration), in bf16 or with the review's V quantization (section
 *     3.4) read as an e4m3 P.V product;
 *   - around them: the SASA augmentation (section 3 "Stage 3", Eqs. 7-10),
 *     the runtime load-balancing planner (section 3 "Stage 2", Eqs. 1-6) and
 *     a window + rotating-anchor mask producer (the LVSA wiki page).
 *
 * Conventions shared by every call
 *   - Q, K, V, O: [B, N, H, d] row-major (d fastest), N = T*Hs*Ws tokens in
 *     raster order (frame, row, column).  d (head_dim) is 64 or 128.
 *   - Blocks: the tokens are reordered (frame-major 2-D Hilbert order, or
 *     identity) and cut into nb = ceil(N / block) blocks of `block` tokens;
 *     the last block holds N - (nb-1)*block tokens.  block is 64 or 128.
 *   - Mask rows: r = (b*H + h)*nb + i, i a query block; columns j are key
 *     blocks of the same order.  A mask is CSR: row_ptr int32 [rows+1]
 *     (row_ptr[0] = 0, non-decreasing), col_idx int32 [nnz], columns unique
 *     and in [0, nb).  Routed masks list each row's columns in importance
 *     order (descending block mass); user masks may use any order.
 *   - Pointers named q, k, v, o, row_ptr, col_idx, L_h, nnz, workspace are
 *     DEVICE pointers on the plan's device, 16-byte aligned (workspace:
 *     256-byte aligned).  The caller owns all of them.  `stream` is a
 *     cudaStream_t (NULL = legacy default stream).
 *   - Every call returns BSA_OK or a negative status.  Argument errors are
 *     reported before anything is launched.  Launches are asynchronous on
 *     `stream`: faults found by the kernels themselves (a malformed mask, a
 *     too-small col_cap, an expired bounded wait) are recorded in the plan's
 *     device error word and read with bsa_last_device_error; no kernel traps.
 *   - A plan may be used from one stream at a time (its device error word
 *     and the workspace are per call).
 */
#ifndef BSA_H
#define BSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ---- */
#define BSA_OK            0
#define BSA_EINVAL       -1   /* bad argument (null/unaligned pointer, p outside (0,1], ...) */
#define BSA_EUNSUPPORTED -2   /* valid but unsupported shape, or not an sm_100 device */
#define BSA_ECAPACITY    -3   /* routed nnz exceeded col_cap (device-detected) */
#define BSA_EWORKSPACE   -4   /* workspace missing, too small or misaligned */
#define BSA_ECUDA        -5   /* a CUDA runtime call or launch failed */
#define BSA_EDEVICE      -6   /* a kernel found malformed input or a bounded wait expired */

/* ---- token orders ---- */
#define BSA_ORDER_HILBERT2D_FRAME 0   /* frames in time order; 2-D Hilbert curve inside each frame */
#define BSA_ORDER_IDENTITY        1   /* raster order */

/* ---- input dtypes for routing ---- */
#define BSA_BF16 0
#define BSA_F32  1

/* ---- workspace queries ---- */
#define BSA_OP_ROUTE 0
#define BSA_OP_ATTN  1
#define BSA_OP_MASK  2
#define BSA_OP_AUGMENT 3

/* ---- attention work-list schedules (bsa_plan_set_schedule) ---- */
#define BSA_SCHED_L2_HEADS       0   /* head groups sized to L2, heaviest group first, heaviest items first */
#define BSA_SCHED_HEAVIEST_FIRST 1   /* every item by descending key-block count */
#define BSA_SCHED_IN_ORDER       2   /* items in row order */

typedef struct bsa_plan bsa_plan;

/*
 * Create a plan for one attention shape on the current CUDA device.
 * Builds the token permutation (perm[n'] = raster index at reordered
 * position n') on the host and keeps it, and a device error word, on the
 * device.  Order BSA_ORDER_HILBERT2D_FRAME follows the FVAttn review, section
 * 3.1 (Hilbert curve block reordering); inside a frame the cells follow the
 * classic 2-D Hilbert curve over the smallest 2^m square covering Hs x Ws
 * (x = column, y = row, starting at (0,0), ending at (2^m-1, 0)), skipping
 * cells outside the grid.
 * Returns BSA_EINVAL / BSA_EUNSUPPORTED for bad shapes (checked before any
 * CUDA call), BSA_ECUDA if the device allocation fails.  *out is NULL on error.
 * Ownership: the plan owns its host struct and device tables; free with
 * bsa_plan_destroy.
 */
int bsa_plan_create(bsa_plan** out, int B, int H, int T, int Hs, int Ws,
                    int head_dim, int block, int order);
void bsa_plan_destroy(bsa_plan* plan);

/* Host-only shape query: N tokens, nb blocks per head, rows = B*H*nb. */
int bsa_plan_info(const bsa_plan* plan, int64_t* N, int64_t* nb, int64_t* rows);

/*
 * Host-only: choose the order in which the attention kernel's persistent CTAs
 * take the work items (b, h, i); it changes the speed, never the result.  It
 * is the single-GPU form of the FVAttn review's runtime load balancing
 * (section 3 "Stage 2" and section 3.2: the heavy heads set the critical
 * path): the balance is across the kernel's CTAs instead of across ranks.
 *   BSA_SCHED_L2_HEADS (the default): heads are cut into groups whose K and V
 *     tiles take at most 40 % of the device's L2; groups run in descending
 *     total work and the items of a group in descending key-block count, so
 *     the CTAs that run at the same time share the tiles of a few heads;
 *   BSA_SCHED_HEAVIEST_FIRST: every item in descending count (over all heads);
 *   BSA_SCHED_IN_ORDER: rows in index order.
 * Takes effect at the next bsa_attn_prepare / bsa_attn_prepare_fp8v.
 * BSA_EINVAL for an unknown schedule.
 */
int bsa_plan_set_schedule(bsa_plan* plan, int schedule);

/*
 * Host-only: the bound, in nanoseconds, of every wait the attention kernels
 * make inside their main loops (a pipeline stage waiting for a tile, an MMA
 * or the softmax of another role); 4e9 (4 s) by default.  A wait that runs
 * out records BSA_EDEVICE in the plan's error word and the kernel stops
 * early; the output of that call is then unspecified, and the CTAs still
 * wait for their own tile copies and MMAs before they exit, so the device
 * stays usable and later calls work normally.  0 makes every wait that is not
 * already satisfied run out at once (for testing that path).  Takes effect at
 * the next bsa_attn_run / bsa_attn_run_fp8v / bsa_sparse_attn call.
 */
int bsa_plan_set_wait_limit(bsa_plan* plan, uint64_t ns);

/*
 * Host-only: the single-GPU analogue of the review's imbalance factor (Eq.
 * 2, rho = max load / mean load) for one work list: the load of a CTA is
 * the number of key blocks of the items the attention kernel assigns to it
 * (one CTA per SM; item k*grid + c goes to CTA c on even rounds k and to
 * CTA grid - 1 - c on odd rounds, grid = min(SM count, rows)).  row_ptr:
 * the mask's row_ptr; work: the work list of a prepared attention workspace
 * (bsa_attn_intermediates), both copied to HOST memory.  *rho, and the
 * largest and mean CTA loads when not NULL.  BSA_EINVAL for null pointers or
 * an invalid work list.
 */
int bsa_schedule_balance(const bsa_plan* plan, const int32_t* row_ptr, const int32_t* work, double* rho,
                         int64_t* max_blocks, double* mean_blocks);

/*
 * Host-only: write the token permutation of a (T, Hs, Ws) grid under `order`
 * into perm[0 .. T*Hs*Ws) (caller-owned host memory).  No CUDA call.
 */
int bsa_token_order(int T, int Hs, int Ws, int order, int32_t* perm);

/* Bytes of device workspace that bsa_route (BSA_OP_ROUTE), bsa_sparse_attn
 * and bsa_sparse_attn_fp8v (BSA_OP_ATTN), bsa_mask_window_anchor and
 * bsa_mask_stripes_device (BSA_OP_MASK) or bsa_augment (BSA_OP_AUGMENT) need; 0 for a NULL plan or
 * an unknown op. */
size_t bsa_workspace_size(const bsa_plan* plan, int op);

/*
 * Top-p block routing (the pages' Stage 1).  Per row r = (b,h,i):
 *   Qbar_i, Kbar_j = means of Q, K over the real tokens of block i, j
 *                    (fp64 sums of the input values);
 *   s_ij = <Qbar_i, Kbar_j> / sqrt(d);  P_ij = softmax_j s_ij   (fp64);
 *   order j by P descending (equal P: ascending j);
 *   n_p  = smallest n whose cumulative mass reaches p (n_p = nb if p >= 1 or
 *          if no prefix reaches p);
 *   n_i  = min(nb, max(k_floor, n_p)) (the Top-k safety floor);
 *   row r of the CSR = the first n_i blocks of that order.
 * Outputs (device): row_ptr int32 [rows+1]; col_idx int32 [col_cap];
 * L_h float [B*H] = (sum_i n_i) / nb (the review's Eq. 1); nnz int64 [1].
 * q, k: [B,N,H,d] of `dtype` (BSA_BF16 or BSA_F32).  p in (0, 1];
 * k_floor >= 0.  col_cap = B*H*nb*nb can never overflow; if the routed nnz
 * exceeds col_cap the columns past col_cap are dropped and the device error
 * word becomes BSA_ECAPACITY.  Needs nb <= 8192 (BSA_EUNSUPPORTED otherwise).
 * workspace: >= bsa_workspace_size(plan, BSA_OP_ROUTE) bytes, 256-aligned.
 */
int bsa_route(const bsa_plan* plan, const void* q, const void* k, int dtype,
              float p, int k_floor,
              int32_t* row_ptr, int32_t* col_idx, int64_t col_cap,
              float* L_h, int64_t* nnz,
              void* workspace, size_t ws_bytes, void* stream);

/*
 * bsa_route without a workspace argument, for callers that cannot allocate
 * device memory at the time they route, such as a host whose device memory is
 * all owned by its own arena or caching allocator.  The FVAttn pages have
 * no counterpart to this call; it only changes where the scratch lives.
 * Same arguments, results and errors as bsa_route.  The scratch is one
 * library-owned device array of 32 MiB, held by every GPU that loads the
 * library until the process exits; plans whose bsa_workspace_size(plan,
 * BSA_OP_ROUTE) exceeds it are rejected with BSA_EWORKSPACE (e.g. the 480p
 * shape fits, the 720p one does not).  The plan's device must be current.
 * The first call on each device looks up the array's device address
 * (cudaGetSymbolAddress) and caches it.  The cached address belongs to the
 * device's primary context: after cudaDeviceReset (or anything else that
 * destroys that context) it is stale, so do not call bsa_route_static again
 * in the same process after such a reset.  All calls share the one array:
 * calls that overlap on the GPU (two streams, or two threads) race and must
 * be serialised by the caller.  Nothing in the array needs to start at zero.
 * Allocates nothing.
 */
int bsa_route_static(const bsa_plan* plan, const void* q, const void* k, int dtype,
                     float p, int k_floor,
                     int32_t* row_ptr, int32_t* col_idx, int64_t col_cap,
                     float* L_h, int64_t* nnz, void* stream);

/*
 * Device pointers to the intermediates the last bsa_route left in
 * `workspace`: pooled Qbar and Kbar, fp64 [B*H, nb, d]; block scores
 * s_ij, fp64 [B*H, nb, nb].  For tests and diagnostics; no CUDA call.
 */
int bsa_route_intermediates(const bsa_plan* plan, void* workspace,
                            const double** qbar, const double** kbar,
                            const double** scores);

/*
 * Device pointer to the full key-block importance order the last bsa_route
 * left in `workspace`: uint16 [rows, nb],
 * row r = every key block of the row in descending block mass (equal mass:
 * ascending j) -- the review's Stage-1 "key-block importance order" output.
 * The first n_i entries of a row are its routed columns.  Valid until the next
 * routing call on the same workspace.  No CUDA call.
 */
int bsa_route_order(const bsa_plan* plan, void* workspace, const uint16_t** order);

/*
 * Slack-aware augmentation, the in-place step of the review's SASA (section 3
 * "Stage 3" and its algorithm flow): every query block of head bh keeps its
 * routed blocks and gains the next extra[bh] blocks of its importance order
 * (clamped at nb); no re-scoring, no re-sorting.  row_ptr: the routed CSR's
 * row_ptr (its counts are the routed prefixes of `order`); order: from
 * bsa_route_order; extra: int32 [B*H] on the device (values < 0 act as 0).
 * Outputs: a new CSR (row_ptr_out [rows+1], col_idx_out [col_cap], columns in
 * importance order), L_h_out [B*H] (Eq. 1) and nnz_out [1]; BSA_ECAPACITY in
 * the device error word if nnz_out > col_cap.  workspace: >=
 * bsa_workspace_size(plan, BSA_OP_AUGMENT) bytes, 256-aligned.
 */
int bsa_augment(const bsa_plan* plan, const int32_t* row_ptr, const uint16_t* order, const int32_t* extra,
                int32_t* row_ptr_out, int32_t* col_idx_out, int64_t col_cap, float* L_h_out,
                int64_t* nnz_out, void* workspace, size_t ws_bytes, void* stream);

/*
 * Host-only: the review's SASA budget for R ranks with workloads L_r (Eqs.
 * 7-10): dL_r = max L - L_r; B_r = n1 * dL_r if dL_r > n2 * max L, else 0
 * (the pages use n1 = 0.8, n2 = 0.07); L_aug_r = L_r + B_r; *A = max(0,
 * max L_aug - max L) + S (the visible overhead).  When heads_per_rank is not
 * NULL, extra_per_head (sum of heads_per_rank entries) receives
 * floor(B_r / heads_per_rank[r]) for each head of rank r, in rank order -- the
 * per-head input of bsa_augment.  Host pointers; no CUDA call.
 */
int bsa_sasa_budget(int R, const float* L_r, float n1, float n2, float S, float* B_r, float* L_aug, float* A,
                    const int32_t* heads_per_rank, int32_t* extra_per_head);

/*
 * Host-only: the runtime load-balancing plan of the review (section 3 "Stage
 * 2", Eqs. 1-6, section 3.2 and its RLB algorithm flow) for R ranks holding
 * n_heads heads: head h lives on rank head_rank[h] and carries workload L_h[h]
 * (Eq. 1; e.g. bsa_route's L_h, all-gathered).  A plan is a set of disjoint
 * rank pairs, each swapping one head of each side (one send and one receive
 * per rank, at most one local head moved); the empty plan is allowed.  The
 * returned plan minimises (max_r L_r_new, Var_r L_r_new) lexicographically
 * (Eq. 6) with L_r_new from Eq. 5, deterministically, so every rank computes
 * the same plan from the same inputs.  moves: int32 [3*R] receives
 * *n_moves triples (src rank, dst rank, head); L_r_new: float [R];
 * rho_before / rho_after (may be NULL): Eq. 2.  R <= 12 (BSA_EUNSUPPORTED
 * above); host pointers; no CUDA call.
 */
int bsa_rlb_plan(int R, int n_heads, const int32_t* head_rank, const float* L_h, int32_t* moves,
                 int* n_moves, float* L_r_new, float* rho_before, float* rho_after);

/*
 * Host-only: per-rank workloads and the imbalance factor of a head placement
 * (FVAttn review, section 3 "Stage 2", Eqs. 1-2): L_r[r] = sum of L_h[h] over
 * the heads with head_rank[h] == r, *rho = max_r L_r / mean_r L_r (1 when
 * every load is 0).  heads_per_rank (int32 [R], may be NULL) receives the
 * number of heads each rank holds.  rho may be NULL.  BSA_EINVAL for R < 1,
 * n_heads < 0, null arrays, a rank outside [0, R) or a negative workload.
 * Host pointers; no CUDA call.
 */
int bsa_rank_loads(int R, int n_heads, const int32_t* head_rank, const float* L_h, float* L_r, float* rho,
                   int32_t* heads_per_rank);

/*
 * Host-only: the review's gain model for a migration plan (section 3 "Stage
 * 2", Eqs. 3-4, and the joint form of Eq. 11): the straggler time saved
 * K = c * (max_r L_r - max_r L_r_new), with c the time per unit of workload,
 * and the net gain G = K - P - C - A, with P the communication cost of
 * moving the migrated heads' state, C the scheduling cost of solving the
 * migration plan and A the slack-augmentation cost (0
 * without augmentation; the pages give no values for c, P, C or A).  L_r,
 * L_r_new: [R] host arrays (e.g. from bsa_rlb_plan).  Negative status for
 * R < 1, null pointers or negative loads.
 */
int bsa_rlb_gain(int R, const float* L_r, const float* L_r_new, double c, double P, double C, double A,
                 double* K, double* G);

/*
 * Host-only: the review's piecewise enabling policy (section 3.3): 0 = do
 * nothing (rho < k1), 1 = slack augmentation only (k1 <= rho < k2), 2 = load
 * balancing then augmentation (rho >= k2); the pages use k1 = 1.05, k2 = 1.10.
 * Negative status for invalid arguments.
 */
int bsa_balance_policy(float rho, float k1, float k2);

/*
 * Fixed mask on the device: a local window plus rotating global anchors (the
 * LVSA wiki page, "TL;DR" and "Key points": a structured local window pattern
 * plus global anchor blocks that shift across diffusion timesteps; the page
 * gives no sizes).  Row (b,h,i) keeps key block j when the latent-frame
 * ranges of blocks i and j (frame-major token order) come within
 * radius_frames frames, plus the anchors {(step + m*floor(nb/n_anchor)) mod
 * nb : m < n_anchor}; columns ascending and unique, identical for every head.
 * radius_frames >= 0, 0 <= n_anchor <= 64, step >= 0.  Outputs as for
 * bsa_route (row_ptr [rows+1], col_idx [col_cap], nnz [1]; BSA_ECAPACITY in
 * the device error word if nnz > col_cap).  workspace: >=
 * bsa_workspace_size(plan, BSA_OP_MASK) bytes, 256-aligned.
 */
int bsa_mask_window_anchor(const bsa_plan* plan, int radius_frames, int n_anchor, int step,
                           int32_t* row_ptr, int32_t* col_idx, int64_t col_cap, int64_t* nnz,
                           void* workspace, size_t ws_bytes, void* stream);

/*
 * Host-only: periodic diagonal stripe block masks (PSA pages: section 3.1,
 * section 3.2, appendix C.2 and appendix D: per-head masks of an inter-frame
 * and an intra-frame stripe family, each with a width, an offset and a
 * stride, an infinite stride being a single diagonal, applied per block).
 * params: host int32 [H][6] = (w_t, o_t, s_t, w_s, o_s, s_s): half-width
 * (>= 0), offset and stride (<= 0: infinite) over latent-frame offsets and
 * over row offsets inside a frame.  A family keeps key offset delta (key
 * minus query) when |delta - o - n*s| <= w for some integer n; query block i
 * and key block j (blocks of `order`, see bsa_plan_create) are kept together
 * when the inter-frame family keeps some frame offset between their frame
 * ranges and the intra-frame family some row offset between their row ranges.
 * Outputs in HOST memory, rows r = (b*H + h)*nb + i as for bsa_route:
 * row_ptr int32 [B*H*nb+1], col_idx int32 [col_cap] (columns ascending),
 * nnz = the full count; BSA_ECAPACITY (columns past col_cap dropped) if nnz
 * > col_cap.  block 64 or 128.  No CUDA call; upload the CSR for
 * bsa_sparse_attn.
 */
int bsa_mask_stripes(int B, int H, int T, int Hs, int Ws, int block, int order, const int32_t* params,
                     int32_t* row_ptr, int32_t* col_idx, int64_t col_cap, int64_t* nnz);

/*
 * The same stripe masks produced on the device, for a plan (the plan's B, H,
 * token order, block and grid; PSA pages, section 3.2 "Efficient and Flexible
 * Kernel": the masks are applied per block inside the attention kernel's
 * pipeline, so here they are written straight into device memory).  params:
 * HOST int32 [H][6] as for bsa_mask_stripes, H <= 160 (BSA_EUNSUPPORTED
 * above), copied into the launch.  Outputs: DEVICE row_ptr int32 [rows+1],
 * col_idx int32 [col_cap] (columns ascending), nnz int64 (device) = the full
 * count; BSA_ECAPACITY in the device error word if it exceeds col_cap
 * (columns past col_cap are dropped).  workspace: >= bsa_workspace_size(plan,
 * BSA_OP_MASK) bytes, 256-aligned.  Identical CSR to bsa_mask_stripes.
 */
int bsa_mask_stripes_device(const bsa_plan* plan, const int32_t* params, int32_t* row_ptr, int32_t* col_idx,
                            int64_t col_cap, int64_t* nnz, void* workspace, size_t ws_bytes, void* stream);

/*
 * Block-sparse attention (the pages' "Block-Sparse Attention Execution"):
 *   O[b, n, h, :] = sum over the real tokens t of the key blocks listed in
 *   row (b,h,i) of softmax_t(Q[b,n,h,:] . K[b,t,h,:] / sqrt(d)) V[b,t,h,:]
 * for every token n of query block i, non-causal, written back in raster
 * token order.  Rows with no key block produce zeros.
 * q, k, v, o: bf16 [B,N,H,d]; row_ptr/col_idx: a CSR mask as above.
 * Equivalent to bsa_attn_prepare followed by bsa_attn_run on `stream`.
 * A column outside [0, nb) is recorded as BSA_EDEVICE in the device error
 * word and the output rows of its query block are then unspecified (every
 * other row is still computed); a decreasing row_ptr counts as an empty row
 * and is recorded the same way.
 * workspace: >= bsa_workspace_size(plan, BSA_OP_ATTN) bytes, 256-aligned.
 */
int bsa_sparse_attn(const bsa_plan* plan, const void* q, const void* k, const void* v,
                    const int32_t* row_ptr, const int32_t* col_idx, void* o,
                    void* workspace, size_t ws_bytes, void* stream);

/*
 * The two halves of bsa_sparse_attn, for callers that time or overlap them.
 * prepare: orders the work items (b,h,i) in the plan's schedule
 *   (bsa_plan_set_schedule), and copies Q, K, V into reordered, zero-padded
 *   [B, H, nb*block, d] bf16 tiles inside the workspace.
 * run: the persistent tcgen05 attention kernel over that work list (for
 *   block 128: two softmax warp groups on alternating key blocks, QK and PV
 *   issued by separate threads; for block 64: one group splitting each row
 *   in halves); writes O.
 * run must follow prepare on the same stream with the same workspace.
 */
int bsa_attn_prepare(const bsa_plan* plan, const void* q, const void* k, const void* v,
                     const int32_t* row_ptr, void* workspace, size_t ws_bytes, void* stream);
int bsa_attn_run(const bsa_plan* plan, const int32_t* row_ptr, const int32_t* col_idx,
                 void* o, void* workspace, size_t ws_bytes, void* stream);

/*
 * Block-sparse attention with an FP8 P.V product (the review's section 3
 * "Block-Sparse Attention Execution" and section 3.4 quantize V before
 * attention; the format is not stated).  Q.K^T stays bf16.  V of each head
 * is scaled per channel, sigma_c = amax over the N tokens of |V[:, c]| / 448,
 * and rounded to e4m3 (OCP E4M3, nearest-even, saturating); the softmax
 * probabilities enter the product as e4m3(16 P) with P taken relative to a
 * running maximum that lags the true one by less than 2^4; products are
 * summed in fp32 and output column c is scaled by sigma_c.  Expected error
 * against exact attention: about 3 % mean relative (two roundings of 2^-4
 * relative each); the tests hold it to 6 %.
 * Same arguments, layouts and error behaviour as bsa_sparse_attn; block 128
 * only (BSA_EUNSUPPORTED otherwise).  The e4m3 V tiles and the scales live in
 * the attention workspace: run_fp8v must follow prepare_fp8v on the same
 * workspace (bsa_attn_run after prepare_fp8v reads them as bf16: undefined).
 */
int bsa_sparse_attn_fp8v(const bsa_plan* plan, const void* q, const void* k, const void* v,
                         const int32_t* row_ptr, const int32_t* col_idx, void* o,
                         void* workspace, size_t ws_bytes, void* stream);
int bsa_attn_prepare_fp8v(const bsa_plan* plan, const void* q, const void* k, const void* v,
                          const int32_t* row_ptr, void* workspace, size_t ws_bytes, void* stream);
int bsa_attn_run_fp8v(const bsa_plan* plan, const int32_t* row_ptr, const int32_t* col_idx,
                      void* o, void* workspace, size_t ws_bytes, void* stream);

/*
 * Host-only: device addresses of the pieces of a prepared attention
 * workspace, for inspection: the work list (int32 [rows], row indices in
 * the order the kernel takes them), the e4m3 V tiles of the FP8 variant
 * (bytes [B*H*nb*d, 128]: per (head, key block) d rows of 128 keys) and
 * their per-channel scales (float [B*H*d]).  Any output may be NULL.
 */
int bsa_attn_intermediates(const bsa_plan* plan, void* workspace, const int32_t** work, const void** v_e4m3,
                           const float** v_scale);

/*
 * Same contract as bsa_attn_run, computed by a slow CUDA-core kernel (one
 * warp per query token, fp32 online softmax).  A cross-check for the
 * tensor-core kernel in tests; not a performance path.
 */
int bsa_attn_run_simt(const bsa_plan* plan, const int32_t* row_ptr, const int32_t* col_idx,
                      void* o, void* workspace, size_t ws_bytes, void* stream);

/*
 * Synchronise `stream`, then read and clear the plan's device error word.
 * Returns BSA_OK, or the first device-side status recorded since the last
 * call (BSA_ECAPACITY, BSA_EDEVICE), or BSA_ECUDA if the stream itself
 * reports an error.
 */
int bsa_last_device_error(const bsa_plan* plan, void* stream);

/* Static description of a status code. */
const char* bsa_strerror(int status);

#ifdef __cplusplus
}
#endif
#endif /* BSA_H */
