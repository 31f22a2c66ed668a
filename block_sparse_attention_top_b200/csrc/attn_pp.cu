// Persistent block-sparse attention, two softmax warp groups in ping-pong
// (FVAttn review, section 3 "Block-Sparse Attention Execution": attention over
// the retained key blocks only, outputs restored to token order).
//
// One CTA per SM walks a static zig-zag share of the heaviest-first work list
// (one item = one 128-row query tile of one head).  The retained key blocks of
// all of a CTA's items form one sequence t = 0, 1, 2, ...; block t belongs to
// softmax group t & 1, so while one group exponentiates block t the other
// loads, reduces and exponentiates block t + 1, and the MUFU/FMA pipes and
// the tensor pipe stay busy across the handshakes.
//
//   warps 0-3   softmax group 0 (one warp per TMEM lane quadrant; one thread
//   warps 4-7   softmax group 1  owns a whole query row of S, O and P)
//   warp 8      QK issuer (1 thread): S[t&1] = Q K_t^T (Q and K from
//               shared memory; the Q tile stays there for the whole item)
//   warp 9      TMA (1 thread): Q tile per item, K_t into a 3-stage ring
//   warp 10     TMA (1 thread): V_t into a 2-stage ring
//   warp 11     PV issuer (1 thread): O (+)= P_t V_t (P_t in TMEM buffer t&1)
//
// QK and PV touch disjoint TMEM columns, so they are issued by two threads:
// a thread that has just issued MMAs stalls on its next shared-memory access
// until the tensor core has taken them, and with one issuer that stall sat
// between every QK and PV.  With two, each stall delays only its own role
// while the tensor pipe works on the other's MMAs.
//
// TMEM: S0 [0,128) S1 [128,256) O [256,256+D) P0, P1 (64 columns each).
// Each group has its own S and P buffer: it releases S as soon as it has
// loaded S_t into registers, so the next QK into that buffer starts while the
// group still works on block t, and it writes P_t while PV_{t-1} (the other
// group's P) may still be running, so consecutive PVs are not separated by a
// softmax handshake.
//
// Online softmax in the log2 domain with the running maximum carried from
// group to group through shared memory: block t reads the maximum m_{t-1} and
// the row sum l_{t-1} published by block t-1 (per-quadrant mbarriers, phases
// strictly alternating between the groups) and publishes m_t, l_t.  m_t is
// published after block t's exponentials, so the groups take turns on the
// exponentials while the other group loads, reduces and stores (measured
// slightly faster than publishing it before them and letting both groups
// exponentiate at once).  A parity
// wait cannot tell a phase from the one two before it, so every wait targets
// a phase at most one past the last phase its waiter knows to be complete.  O is
// rescaled in TMEM only when the maximum grows by more than 2^8 (after PV_{t-1}
// is done and before P_t is released; only then does a group wait for the
// other group's PV).  The group that owns an item's last
// block writes O / l in bf16 to the tokens' raster positions (the inverse
// token permutation fused into the store), then frees O for the next item.
//
// A column outside [0, nb) is recorded as BSA_EDEVICE and replaced by the
// nearest valid block, so every role still walks the same sequence.
//
// FP8 variant (F8 = true; the review's V quantization, format not stated):
// V arrives as e4m3 tiles [d x 128 keys] per (head, key block) with per-
// channel scales sigma_c (quant.cu); the probabilities enter as e4m3(16 P)
// with P relative to the running maximum, which is rescaled once it grows by
// more than 2^4 (so 16 P <= 256 fits e4m3), PV is a kind::f8f6f4 MMA with
// fp32 accumulation, and the epilogue writes O[:, c] * sigma_c / l.
//
// Every wait on an mbarrier in the main loops spins on test_wait and is
// bounded (the plan's wait limit, 4 s by default); on expiry the CTA records
// BSA_EDEVICE and raises a shared abort flag that stops the other roles.
// Before TMEM is freed and the CTA returns, each TMA thread waits (with a
// fixed 4 s bound) until every tile it issued has landed and each MMA thread
// until its MMAs are complete.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "bsa_internal.cuh"
#include "tc_common.cuh"

namespace bsa {
namespace {

using namespace tc;

constexpr int kBlk = 128;                 // query rows per tile = key tokens per block
constexpr int kGroupWarps = 4;            // one warp per TMEM lane quadrant
constexpr int kMmaWarp = 2 * kGroupWarps, kKWarp = kMmaWarp + 1, kVWarp = kMmaWarp + 2, kPvWarp = kMmaWarp + 3;
constexpr int kThreads = 32 * (kPvWarp + 1);
constexpr int kGroupThreads = 32 * kGroupWarps;
constexpr int kKStages = 3, kVStages = 2;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO = 256;
constexpr int kPolyPairs = 0;             // pairs in every 8 exponentiated on the FMA pipe (0: all on
                                          // MUFU; 1 and 2 measured 12-18 % slower in this kernel)

template <int D, bool F8>
struct PPLayout {
    static constexpr uint32_t kColP = kColO + D;            // P0; P1 follows
    static_assert(kColP + 2 * (kBlk / 2) <= kTmemCols, "TMEM budget");
    static constexpr int kTile = kBlk * D * 2;      // one Q, K or V tile: D/64 slabs of [128 rows x 128 B]
    static constexpr int kVTile = F8 ? D * 128 : kTile;   // e4m3 V: [D rows x 128 B] (keys along a row)
    static constexpr int offQ = 0;
    static constexpr int offK = offQ + kTile;
    static constexpr int offV = offK + kKStages * kTile;
    static constexpr int offPub = offV + kVStages * kVTile;  // float m[2][128], l[2][128]
    static constexpr int offBar = offPub + 4 * kBlk * 4;
    static constexpr int kBars = 40;
    static constexpr int offMisc = offBar + kBars * 8;
    static constexpr int kBytes = offMisc + 64;
    static constexpr int kAlloc = kBytes + 1024;   // room to align the base to 1024 B
};
enum {
    Q_FULL = 0, Q_EMPTY, K_FULL0, K_EMPTY0 = K_FULL0 + kKStages, V_FULL0 = K_EMPTY0 + kKStages,
    V_EMPTY0 = V_FULL0 + kVStages, S_FULL0 = V_EMPTY0 + kVStages, S_FREE0 = S_FULL0 + 2, P_FULL0 = S_FREE0 + 2,
    PV_DONE0 = P_FULL0 + 2, O_DONE = PV_DONE0 + 2, O_FREE, M_PUB0, L_PUB0 = M_PUB0 + 8, DRAIN_QK = L_PUB0 + 8, DRAIN_PV, NBARS
};
static_assert(NBARS <= 40, "barrier slots");

struct Params {
    const int32_t* row_ptr;
    const int32_t* col_idx;
    const int32_t* work;
    const int32_t* perm;
    __nv_bfloat16* o;
    int32_t* err;
    int N, H, nb, rows;
    int64_t npad;
    float scale_log2;
    const float* sigma;      // F8: per (head, channel) V scale, [B*H, D]
    unsigned long long wait_ns;   // bound of every main-loop wait
};

__device__ __forceinline__ int item_index(int k, int cta, int grid) {
    return k * grid + ((k & 1) ? (grid - 1 - cta) : cta);
}
__device__ __forceinline__ int clamp_col(int j, int nb) { return j < 0 ? 0 : (j >= nb ? nb - 1 : j); }

// The non-empty items of this CTA and their blocks, in the order every role walks them.
struct Walk {
    int k = 0, r = 0, beg = 0, end = 0, jj = 0, items = 0;
    bool ok = false;
    __device__ void open(const Params& prm, int cta, int grid) {
        for (;;) {
            const int idx = item_index(k, cta, grid);
            if (idx >= prm.rows) { ok = false; return; }
            ++k;
            r = prm.work[idx];
            beg = prm.row_ptr[r];
            end = prm.row_ptr[r + 1];
            if (end > beg) { jj = beg; ++items; ok = true; return; }
        }
    }
    __device__ void next(const Params& prm, int cta, int grid) {
        if (++jj == end) open(prm, cta, grid);
    }
    __device__ bool first() const { return jj == beg; }
    __device__ bool last() const { return jj == end - 1; }
};

// P for one row: p = 2^(s * scale - m) as bf16 pairs, and the row sum.
// kPolyPairs pairs of every 8 go through the FMA-pipe polynomial unless the
// block is ragged (masked keys are -inf there).
template <int N, bool RAGGED>
__device__ __forceinline__ float softmax_row(const uint32_t* s, float scale, float neg_m, uint32_t* pk) {
    float acc[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) acc[u] = 0.f;
#pragma unroll
    for (int c = 0; c < N; c += 2) {
        float x0, x1, p0, p1;
        ffma2(x0, x1, __uint_as_float(s[c]), __uint_as_float(s[c + 1]), scale, scale, neg_m, neg_m);
        if (!RAGGED && ((c / 2) & 7) >= 8 - kPolyPairs) {
            ex2_poly2(x0, x1, p0, p1);
        } else {
            p0 = ex2_mufu(x0);
            p1 = ex2_mufu(x1);
        }
        const int u = (c / 2) & 3;
        fadd2(acc[2 * u], acc[2 * u + 1], acc[2 * u], acc[2 * u + 1], p0, p1);
        pk[c / 2] = pack_bf16(p0, p1);
    }
    return ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
}

// The same for the FP8 product: p (already in units of 16 P) rounded to e4m3,
// four keys to a 32-bit word (key 4w in the low byte), and the row sum.
template <int N, bool RAGGED>
__device__ __forceinline__ float softmax_row_e4m3(const uint32_t* s, float scale, float neg_m, uint32_t* pk) {
    float acc[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) acc[u] = 0.f;
#pragma unroll
    for (int c = 0; c < N; c += 4) {
        float x0, x1, x2, x3;
        ffma2(x0, x1, __uint_as_float(s[c]), __uint_as_float(s[c + 1]), scale, scale, neg_m, neg_m);
        ffma2(x2, x3, __uint_as_float(s[c + 2]), __uint_as_float(s[c + 3]), scale, scale, neg_m, neg_m);
        const float p0 = ex2_mufu(x0), p1 = ex2_mufu(x1), p2 = ex2_mufu(x2), p3 = ex2_mufu(x3);
        const int u = (c / 4) & 3;
        fadd2(acc[2 * u], acc[2 * u + 1], acc[2 * u], acc[2 * u + 1], p0, p1);
        fadd2(acc[2 * u], acc[2 * u + 1], acc[2 * u], acc[2 * u + 1], p2, p3);
        const uint32_t lo = __nv_cvt_float2_to_fp8x2(make_float2(p0, p1), __NV_SATFINITE, __NV_E4M3);
        const uint32_t hi = __nv_cvt_float2_to_fp8x2(make_float2(p2, p3), __NV_SATFINITE, __NV_E4M3);
        pk[c / 4] = lo | (hi << 16);
    }
    return ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
}

template <int D, bool F8, uint32_t kEvery>
__global__ void __launch_bounds__(kThreads, 1)
k_attn_pp(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
          const __grid_constant__ CUtensorMap tmV, const Params prm) {
    using L = PPLayout<D, F8>;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar0 = sbase + L::offBar;
    auto bar = [&](int i) { return bar0 + 8u * (uint32_t)i; };
    volatile WaitCtl* ctl = reinterpret_cast<volatile WaitCtl*>(smem + L::offMisc);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::offMisc + 16);
    float* m_pub = reinterpret_cast<float*>(smem + L::offPub);          // [2][128]
    float* l_pub = m_pub + 2 * kBlk;                                     // [2][128]

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    if (threadIdx.x == 0) {
        ctl->abort = 0;
        ctl->limit_ns = prm.wait_ns;
        for (int i = 0; i < NBARS; ++i) {
            uint32_t count = 1;
            if (i == S_FREE0 || i == S_FREE0 + 1 || i == P_FULL0 || i == P_FULL0 + 1 || i == O_FREE)
                count = kGroupThreads;
            if (i >= M_PUB0 && i < DRAIN_QK) count = 32;
            mbar_init(bar(i), count);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == kMmaWarp) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(tmem_slot)), "r"(kTmemCols) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    fence_before();
    __syncthreads();
    fence_after();
    const uint32_t tmem = *tmem_slot;
    const int grid = gridDim.x, cta = blockIdx.x;
    const int nb = prm.nb;

    if (warp == kKWarp || warp == kVWarp) {
        // ------------------------------------------------------------ producers
        const bool kside = warp == kKWarp;
        if (lane == 0) {
            uint32_t u = 0, q_it = 0;
            bool ok = true;
            Walk w;
            for (w.open(prm, cta, grid); w.ok && ok; w.next(prm, cta, grid), ++u) {
                const int bh = w.r / nb;
                if (kside && w.first()) {
                    if (q_it > 0 && !(ok = mbar_wait<kEvery>(bar(Q_EMPTY), (q_it - 1) & 1, ctl))) break;
                    mbar_expect_tx(bar(Q_FULL), L::kTile);
                    const int i = w.r % nb;
                    for (int s = 0; s < D / 64; ++s)
                        tma_load_2d(sbase + L::offQ + s * kBlk * 128, &tmQ, s * 64,
                                    (int)(bh * prm.npad + (int64_t)i * kBlk), bar(Q_FULL));
                    ++q_it;
                }
                const int j_raw = prm.col_idx[w.jj];
                const int j = clamp_col(j_raw, nb);
                if (kside && j != j_raw) record_error(prm.err, BSA_EDEVICE, w.r);
                const int y = (int)(bh * prm.npad + (int64_t)j * kBlk);
                if (kside) {
                    const int st = u % kKStages;
                    const uint32_t use = u / kKStages;
                    if (use > 0 && !(ok = mbar_wait<kEvery>(bar(K_EMPTY0 + st), (use - 1) & 1, ctl))) break;
                    mbar_expect_tx(bar(K_FULL0 + st), L::kTile);
                    for (int s = 0; s < D / 64; ++s)
                        tma_load_2d(sbase + L::offK + st * L::kTile + s * kBlk * 128, &tmK, s * 64, y,
                                    bar(K_FULL0 + st));
                } else {
                    const int st = u % kVStages;
                    const uint32_t use = u / kVStages;
                    if (use > 0 && !(ok = mbar_wait<kEvery>(bar(V_EMPTY0 + st), (use - 1) & 1, ctl))) break;
                    mbar_expect_tx(bar(V_FULL0 + st), L::kVTile);
                    if constexpr (F8) {
                        // e4m3 tile of (head, block j): rows (bh * nb + j) * D .. + D, 128 keys each
                        tma_load_2d(sbase + L::offV + st * L::kVTile, &tmV, 0, (int)(((int64_t)bh * nb + j) * D),
                                    bar(V_FULL0 + st));
                    } else {
                        for (int s = 0; s < D / 64; ++s)
                            tma_load_2d(sbase + L::offV + st * L::kVTile + s * kBlk * 128, &tmV, s * 64, y,
                                        bar(V_FULL0 + st));
                    }
                }
            }
            if (!ok) { ctl->abort = 1; record_error(prm.err, BSA_EDEVICE, -1); }
            // every tile this thread issued lands before the CTA exits (the last
            // load of each stage completes its phase; nothing is issued after it)
            const uint32_t stages = kside ? kKStages : kVStages;
            for (uint32_t st = 0; st < stages; ++st) {
                const uint32_t loads = u > st ? (u - 1 - st) / stages + 1 : 0;
                if (loads > 0) mbar_drain(bar((kside ? K_FULL0 : V_FULL0) + st), (loads - 1) & 1);
            }
            if (kside && q_it > 0) mbar_drain(bar(Q_FULL), (q_it - 1) & 1);
        }
    } else if (warp == kMmaWarp) {
        // ---------------------------------------------------------- QK issuer
        if (lane == 0) {
            constexpr uint32_t idesc_qk = instr_desc(kBlk, 0);
            Walk qc;
            uint32_t uq = 0, q_it = 0;
            bool ok = true;
            for (qc.open(prm, cta, grid); qc.ok && ok; qc.next(prm, cta, grid), ++uq) {
                if (qc.first()) {                            // this item's Q tile has landed
                    if (!(ok = mbar_wait<kEvery>(bar(Q_FULL), q_it & 1, ctl))) break;
                    ++q_it;
                }
                // S[uq&1] = Q K_uq^T once the group has loaded S_{uq-2} from that buffer
                const int sb = uq & 1;
                if (uq >= 2 && !(ok = mbar_wait<kEvery>(bar(S_FREE0 + sb), ((uq - 2) >> 1) & 1, ctl))) break;
                const int st = uq % kKStages;
                if (!(ok = mbar_wait<kEvery>(bar(K_FULL0 + st), (uq / kKStages) & 1, ctl))) break;
                fence_after();
                const uint32_t d_s = tmem + (sb ? kColS1 : kColS0);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t koff = (kk / 4) * kBlk * 128 + (kk % 4) * 32;
                    mma_ss(d_s, smem_desc(sbase + L::offQ + koff, 16, 1024),
                           smem_desc(sbase + L::offK + st * L::kTile + koff, 16, 1024), idesc_qk, kk > 0 ? 1u : 0u);
                }
                commit(bar(S_FULL0 + sb));
                commit(bar(K_EMPTY0 + st));
                if (qc.last()) commit(bar(Q_EMPTY));         // the Q tile may be replaced
            }
            if (!ok) {
                ctl->abort = 1;
                record_error(prm.err, BSA_EDEVICE, -2);
            }
            // drain: everything this thread issued completes before TMEM is freed
            commit(bar(DRAIN_QK));
            mbar_drain(bar(DRAIN_QK), 0);
        }
    } else if (warp == kPvWarp) {
        // ---------------------------------------------------------- PV issuer
        if (lane == 0) {
            constexpr uint32_t idesc_pv = F8 ? instr_desc_e4m3(D) : instr_desc(D, 1);
            Walk pc;
            uint32_t up = 0;
            bool ok = true;
            for (pc.open(prm, cta, grid); pc.ok && ok; pc.next(prm, cta, grid), ++up) {
                // O (+)= P_up V_up; the first block of an item also waits for the
                // previous item's epilogue to have read O
                if (!(ok = mbar_wait<kEvery>(bar(P_FULL0 + (up & 1)), (up >> 1) & 1, ctl))) break;
                if (pc.first() && pc.items > 1 && !(ok = mbar_wait<kEvery>(bar(O_FREE), (pc.items - 2) & 1, ctl)))
                    break;
                const int st = up % kVStages;
                if (!(ok = mbar_wait<kEvery>(bar(V_FULL0 + st), (up / kVStages) & 1, ctl))) break;
                fence_after();
                const bool fresh = pc.first();
                const uint32_t p_tmem = tmem + L::kColP + (up & 1) * (kBlk / 2);
                if constexpr (F8) {
                    // K = 32 keys (32 bytes) per MMA: P columns kk*8.., V row bytes kk*32..
#pragma unroll
                    for (int kk = 0; kk < kBlk / 32; ++kk) {
                        const uint64_t b = smem_desc(sbase + L::offV + st * L::kVTile + kk * 32, 16, 1024);
                        mma_ts_f8(tmem + kColO, p_tmem + kk * 8, b, idesc_pv, (fresh && kk == 0) ? 0u : 1u);
                    }
                } else {
#pragma unroll
                    for (int kk = 0; kk < kBlk / 16; ++kk) {
                        const uint64_t b = smem_desc(sbase + L::offV + st * L::kVTile + kk * 16 * 128, kBlk * 128, 1024);
                        mma_ts(tmem + kColO, p_tmem + kk * 8, b, idesc_pv, (fresh && kk == 0) ? 0u : 1u);
                    }
                }
                commit(bar(PV_DONE0 + (up & 1)));
                commit(bar(V_EMPTY0 + st));
                if (pc.last()) commit(bar(O_DONE));
            }
            if (!ok) {
                ctl->abort = 1;
                record_error(prm.err, BSA_EDEVICE, -4);
            }
            commit(bar(DRAIN_PV));
            mbar_drain(bar(DRAIN_PV), 0);
        }
    } else {
        // ------------------------------------------------------------- softmax
        const int g = warp / kGroupWarps;                // group: blocks t with t & 1 == g
        const int quad = warp & 3;                       // TMEM lane quadrant
        const int row = 32 * quad + lane;                // TMEM lane == query row in tile
        const uint32_t lane_base = (uint32_t)(32 * quad) << 16;
        const uint32_t s_col = g ? kColS1 : kColS0;
        const int mine = g * kBlk + row, other = (1 - g) * kBlk + row;       // slots in m_pub / l_pub
        const int pub_mine = 4 * g + quad, pub_other = 4 * (1 - g) + quad;   // barrier offsets
        uint32_t t = 0, items = 0;
        bool ok = true;
        for (int k = 0; ok; ++k) {
            const int idx = item_index(k, cta, grid);
            if (idx >= prm.rows) break;
            const int r = prm.work[idx];
            const int beg = prm.row_ptr[r], end = prm.row_ptr[r + 1];
            const int bh = r / nb, i = r % nb;
            const int b = bh / prm.H, h = bh % prm.H;
            const int n_tok = i * kBlk + row;            // reordered position of this row
            const bool row_real = n_tok < prm.N;
            __nv_bfloat16* dst = prm.o + (((int64_t)b * prm.N + (row_real ? prm.perm[n_tok] : 0)) * prm.H + h) * D;
            if (end <= beg) {                            // no key block: zeros, written by the next block's group
                if ((int)(t & 1) == g && row_real)
                    for (int c = 0; c < D / 8; ++c) reinterpret_cast<uint4*>(dst)[c] = make_uint4(0, 0, 0, 0);
                continue;
            }
            ++items;
            for (int jj = beg; jj < end && ok; ++jj, ++t) {
                if ((int)(t & 1) != g) continue;
                const int j = clamp_col(prm.col_idx[jj], nb);
                const bool first = jj == beg, last = jj == end - 1;
                if (!(ok = warp_wait<kEvery>(bar(S_FULL0 + g), (t >> 1) & 1, ctl))) break;
                fence_after();
                uint32_t sv[kBlk];
#pragma unroll
                for (int c = 0; c < kBlk / 32; ++c) tmem_ld32(tmem + lane_base + s_col + c * 32, sv + 32 * c);
                tmem_wait_ld();
                fence_before();
                mbar_arrive(bar(S_FREE0 + g));            // S buffer g may take the next QK
                const int valid_keys = prm.N - j * kBlk;
                const bool ragged = valid_keys < kBlk;
                if (ragged) {
#pragma unroll
                    for (int c = 0; c < kBlk; ++c)
                        if (c >= valid_keys) sv[c] = __float_as_uint(-INFINITY);
                }
                const float mx = row_max<kBlk>(sv, -INFINITY) * prm.scale_log2;
                // running maximum from the previous block (the other group)
                float m_prev = -INFINITY;
                if (t > 0) {
                    if (!(ok = warp_wait<kEvery>(bar(M_PUB0 + pub_other), ((t - 1) >> 1) & 1, ctl))) break;
                    m_prev = m_pub[other];
                }
                float m_use = m_prev, alpha = 1.f;
                bool rescale = false;
                if (first) {
                    m_use = mx;
                } else if (mx > m_prev + (F8 ? 4.f : 8.f)) {
                    alpha = ex2_mufu(m_prev - mx);
                    m_use = mx;
                    rescale = true;
                }
                uint32_t pk[kBlk / 2];
                float rowsum;
                if constexpr (F8) {                          // in units of 16 P: 2^(s*scale - m + 4)
                    rowsum = ragged ? softmax_row_e4m3<kBlk, true>(sv, prm.scale_log2, 4.f - m_use, pk)
                                    : softmax_row_e4m3<kBlk, false>(sv, prm.scale_log2, 4.f - m_use, pk);
                } else {
                    rowsum = ragged ? softmax_row<kBlk, true>(sv, prm.scale_log2, -m_use, pk)
                                    : softmax_row<kBlk, false>(sv, prm.scale_log2, -m_use, pk);
                }
                m_pub[mine] = m_use;                         // the other group's next block may start
                mbar_arrive(bar(M_PUB0 + pub_mine));
                // PV_{t-2} done: this group's P buffer is free.  PVs of odd and even
                // blocks complete on separate barriers and each group waits on every
                // phase of its own (a parity wait on a barrier still a phase behind
                // would match its previous phase).
                if (t >= 2) {
                    if (!(ok = warp_wait<kEvery>(bar(PV_DONE0 + g), ((t - 2) >> 1) & 1, ctl))) break;
                    fence_after();
                }
                const bool any_rescale = __any_sync(0xffffffffu, rescale);
                if (any_rescale) {
                    // O must hold every earlier block before it is rescaled: PV_{t-1}
                    // done.  That barrier's previous phase (PV_{t-3}) has completed, as
                    // PV_{t-2} just did, so this occasional parity wait is exact.
                    if (!(ok = warp_wait<kEvery>(bar(PV_DONE0 + (1 - g)), ((t - 1) >> 1) & 1, ctl))) break;
                    fence_after();
#pragma unroll
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t o[32];
                        tmem_ld32(tmem + lane_base + kColO + c * 32, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                        tmem_st32(tmem + lane_base + kColO + c * 32, o);
                    }
                }
                constexpr int kPCols = F8 ? kBlk / 4 : kBlk / 2;     // 32-bit TMEM columns of one P row
#pragma unroll
                for (int c = 0; c < kPCols / 32; ++c)
                    tmem_st32(tmem + lane_base + L::kColP + g * (kBlk / 2) + c * 32, pk + 32 * c);
                // running row sum
                float l_prev = 0.f;
                if (t > 0) {
                    if (!(ok = warp_wait<kEvery>(bar(L_PUB0 + pub_other), ((t - 1) >> 1) & 1, ctl))) break;
                    l_prev = l_pub[other];
                }
                const float l = first ? rowsum : l_prev * alpha + rowsum;
                l_pub[mine] = l;
                mbar_arrive(bar(L_PUB0 + pub_mine));
                tmem_wait_st();
                fence_before();
                mbar_arrive(bar(P_FULL0 + g));              // per-group barrier: the groups' arrivals
                                                             // for consecutive blocks may overtake
                if (!last) continue;
                // epilogue: the item's last PV, then O / l to the tokens' raster rows
                if (!(ok = warp_wait<kEvery>(bar(O_DONE), (items - 1) & 1, ctl))) break;
                fence_after();
                const float inv = 1.f / l;
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t o[32];
                    tmem_ld32(tmem + lane_base + kColO + c * 32, o);
                    tmem_wait_ld();
                    if constexpr (F8) {                      // per-channel V scale
                        const float* sg = prm.sigma + (int64_t)(r / nb) * D + c * 32;
#pragma unroll
                        for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * __ldg(sg + e));
                    }
                    if (row_real) {
#pragma unroll
                        for (int e = 0; e < 32; e += 8) {
                            uint4 v;
                            v.x = pack_bf16(__uint_as_float(o[e + 0]) * inv, __uint_as_float(o[e + 1]) * inv);
                            v.y = pack_bf16(__uint_as_float(o[e + 2]) * inv, __uint_as_float(o[e + 3]) * inv);
                            v.z = pack_bf16(__uint_as_float(o[e + 4]) * inv, __uint_as_float(o[e + 5]) * inv);
                            v.w = pack_bf16(__uint_as_float(o[e + 6]) * inv, __uint_as_float(o[e + 7]) * inv);
                            *reinterpret_cast<uint4*>(dst + c * 32 + e) = v;
                        }
                    }
                }
                fence_before();
                mbar_arrive(bar(O_FREE));
            }
        }
        if (!ok) { ctl->abort = 1; record_error(prm.err, BSA_EDEVICE, -3); }
        tmem_wait_st();                                  // no TMEM access of this warp outlives the loop
        tmem_wait_ld();
    }

    fence_before();
    __syncthreads();
    fence_after();
    if (warp == kMmaWarp) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
    }
}

template <int D, bool F8, uint32_t kEvery>
cudaError_t launch_t(const bsa_plan& p, const void* qp, const void* kp, const void* vp, const Params& prm,
                     cudaStream_t s) {
    using L = PPLayout<D, F8>;
    const int64_t rows_total = (int64_t)p.B * p.H * p.nb * p.block;
    CUtensorMap mq, mk, mv;
    if (!make_map(&mq, qp, rows_total, D, kBlk) || !make_map(&mk, kp, rows_total, D, kBlk))
        return cudaErrorInvalidValue;
    if (F8 ? !make_map_u8(&mv, vp, (int64_t)p.B * p.H * p.nb * D, D) : !make_map(&mv, vp, rows_total, D, kBlk))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(k_attn_pp<D, F8, kEvery>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         L::kAlloc);
    if (e != cudaSuccess) return e;
    const int grid = (int)std::min<int64_t>(p.num_sms, p.rows);
    k_attn_pp<D, F8, kEvery><<<grid, kThreads, L::kAlloc, s>>>(mq, mk, mv, prm);
    return cudaGetLastError();
}

// a wait limit below a millisecond: the variant that checks it at every probe
template <int D, bool F8>
cudaError_t launch(const bsa_plan& p, const void* qp, const void* kp, const void* vp, const Params& prm,
                   cudaStream_t s) {
    if (prm.wait_ns < 1000000ull) return launch_t<D, F8, 0>(p, qp, kp, vp, prm, s);
    return launch_t<D, F8, 1023>(p, qp, kp, vp, prm, s);
}

}  // namespace

bool attn_pp_supported(const bsa_plan& p) { return p.block == kBlk && (p.d == 128 || p.d == 64); }

cudaError_t launch_attn_pp(const bsa_plan& p, const void* qp, const void* kp, const void* vp,
                           const int32_t* row_ptr, const int32_t* col_idx, const int32_t* work, void* o,
                           const float* sigma, cudaStream_t s) {
    Params prm;
    prm.row_ptr = row_ptr;
    prm.col_idx = col_idx;
    prm.work = work;
    prm.perm = p.d_perm;
    prm.o = (__nv_bfloat16*)o;
    prm.err = p.d_err;
    prm.N = (int)p.N;
    prm.H = p.H;
    prm.nb = (int)p.nb;
    prm.rows = (int)p.rows;
    prm.npad = p.nb * p.block;
    prm.scale_log2 = 1.4426950408889634f / sqrtf((float)p.d);
    prm.sigma = sigma;
    prm.wait_ns = p.wait_ns;
    if (sigma) {                      // e4m3 V tiles at vp, scales at sigma
        if (p.d == 128) return launch<128, true>(p, qp, kp, vp, prm, s);
        return launch<64, true>(p, qp, kp, vp, prm, s);
    }
    if (p.d == 128) return launch<128, false>(p, qp, kp, vp, prm, s);
    return launch<64, false>(p, qp, kp, vp, prm, s);
}

}  // namespace bsa
