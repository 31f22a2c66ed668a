// Persistent block-sparse attention on the 5th-generation tensor cores
// (FVAttn review, section 3 "Block-Sparse Attention Execution": attention
// computed only over the retained key blocks, outputs restored to token order).
//
// One CTA per SM walks a static zig-zag share of the heaviest-first work list
// (one item = one 128-row query tile of one head).  Per item and retained key
// block j, with S, P and O living in tensor memory (TMEM):
//
//   warp 0 (1 thread)   TMA: Q tile once per item; K_j into a 3-stage ring
//   warp 10 (1 thread)  TMA: V_j into a 2-stage ring (runs ahead independently of K)
//   warp 1 (1 thread)   tcgen05.cp: Q tile smem -> TMEM once per item;
//                       tcgen05.mma: S[j%2] = Q K_j^T   (M=128, N=block, K=d; Q in TMEM, K in smem)
//                                    O     += P_j V_j   (M=128, N=d, K=block; P in TMEM, V in smem)
//   warps 2..9          softmax: TMEM lane = query row; each row is split over
//                       two warps, one per half of the key (and output)
//                       columns, which swap their half-row maxima (and at the
//                       end their row sums) through shared memory behind a
//                       bounded per-quadrant mbarrier.  Online softmax in the
//                       log2 domain; one exponential in eight runs as a
//                       polynomial on the FMA pipe to offload the MUFU unit;
//                       P_j overwrites the first half of S_j's TMEM columns as
//                       bf16 pairs (tcgen05.st); the O row is rescaled in TMEM only when
//                       its running max grows by more than 2^8.  Epilogue: the
//                       two partial row sums meet through shared memory, then
//                       O / l, bf16, stored at the token's raster position (the
//                       inverse Hilbert permutation is fused into this store).
//
// S (with P) is double-buffered, so QK^T of block j+1 and PV of block j-1 run
// on the tensor pipe while the softmax warps work on block j.  Keeping Q in
// TMEM halves the shared-memory reads of QK^T, which would otherwise need the
// SM's whole shared-memory bandwidth at full MMA rate.  TMEM columns:
// S0 [0,128) S1 [128,256) O [256,384) Q [384,448).
//
// Every wait on an mbarrier in the main loops spins on test_wait and is
// bounded (the plan's wait limit, 4 s of %globaltimer by default); on expiry
// the CTA records BSA_EDEVICE and raises a shared abort flag that stops the
// other roles.  Before TMEM is freed and the CTA returns, each TMA thread
// waits (with a fixed 4 s bound) until every tile it issued has landed and
// the MMA thread until its MMAs are complete.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include "bsa_internal.cuh"
#include "tc_common.cuh"

namespace bsa {
namespace {

constexpr int kSoftmaxWarps = 8;
constexpr int kThreads = 32 * (3 + kSoftmaxWarps);   // Q/K producer, MMA, softmax x8, V producer
constexpr int kKStages = 3, kVStages = 2;
constexpr int kVWarp = 2 + kSoftmaxWarps;
constexpr int kTileM = 128;                          // query rows per tile (TMEM lanes)
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO = 256, kColQ = 384;

using namespace tc;

// P for this warp's half row: p = 2^(s * scale - m), packed to bf16 pairs, and
// the half-row sum.  One pair in eight goes through the FMA-pipe polynomial
// unless the block is ragged (masked keys are -inf there).
template <int HC, bool RAGGED>
__device__ __forceinline__ float softmax_half(const uint32_t* s, float scale, float neg_m, uint32_t* pk) {
    float acc[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) acc[u] = 0.f;
#pragma unroll
    for (int c = 0; c < HC; c += 2) {
        float x0, x1, p0, p1;
        ffma2(x0, x1, __uint_as_float(s[c]), __uint_as_float(s[c + 1]), scale, scale, neg_m, neg_m);
        if (!RAGGED && (c & 14) == 14) {
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

// ------------------------------------------------------------- shared layout
template <int D, int BLK>
struct Smem {
    static constexpr int kQ = kTileM * D * 2;       // Q tile: D/64 slabs of [128 rows x 128 B]
    static constexpr int kKV = BLK * D * 2;         // one K or V tile: D/64 slabs of [BLK rows x 128 B]
    static constexpr int offQ = 0;
    static constexpr int offK = offQ + kQ;
    static constexpr int offV = offK + kKStages * kKV;
    // float [2 kv parity][2 half][128 rows] half-row maxima, then the same for row sums by item parity
    static constexpr int offXchg = offV + kVStages * kKV;
    static constexpr int offBar = offXchg + 2 * 2 * 2 * kTileM * 4;
    static constexpr int kBars = 24;
    static constexpr int offMisc = offBar + kBars * 8;
    static constexpr int kBytes = offMisc + 64;
    static constexpr int kAlloc = kBytes + 1024;   // room to align the base to 1024 B
};
// barrier slots
enum { B_QFULL = 0, B_QEMPTY, B_KFULL0, B_KEMPTY0 = B_KFULL0 + kKStages, B_VFULL0 = B_KEMPTY0 + kKStages,
       B_VEMPTY0 = B_VFULL0 + kVStages, B_SFULL0 = B_VEMPTY0 + kVStages, B_SFULL1, B_PFULL, B_PVDONE, B_DRAIN,
       B_PAIR0, B_PAIR1, B_PAIR2, B_PAIR3, B_COUNT };

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
    unsigned long long wait_ns;   // bound of every main-loop wait
};

// Work item sequence of this CTA: zig-zag over the heaviest-first list.
__device__ __forceinline__ int item_index(int k, int cta, int grid) {
    return k * grid + ((k & 1) ? (grid - 1 - cta) : cta);
}

__device__ __forceinline__ bool valid_col(int j, int nb) { return j >= 0 && j < nb; }

template <int D, int BLK, uint32_t kEvery>
__global__ void __launch_bounds__(kThreads, 1)
k_attn_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
          const __grid_constant__ CUtensorMap tmV, const Params prm) {
    using L = Smem<D, BLK>;
    constexpr int HC = BLK / 2;     // S columns per softmax warp
    constexpr int OC = D / 2;       // O columns per softmax warp
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar0 = sbase + L::offBar;
    auto bar = [&](int i) { return bar0 + 8u * (uint32_t)i; };
    volatile WaitCtl* ctl = reinterpret_cast<volatile WaitCtl*>(smem + L::offMisc);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::offMisc + 16);
    float* xchg = reinterpret_cast<float*>(smem + L::offXchg);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

    if (threadIdx.x == 0) {
        ctl->abort = 0;
        ctl->limit_ns = prm.wait_ns;
        for (int i = 0; i < B_COUNT; ++i)
            mbar_init(bar(i), i == B_PFULL ? 32u * kSoftmaxWarps : (i >= B_PAIR0 ? 64u : 1u));
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (BLK < kTileM) {
        // rows BLK..127 of the Q tile are never loaded: keep them zero
        for (int s = 0; s < D / 64; ++s)
            for (int e = threadIdx.x; e < (kTileM - BLK) * 128 / 16; e += kThreads)
                reinterpret_cast<uint4*>(smem + L::offQ + s * kTileM * 128 + BLK * 128)[e] = make_uint4(0, 0, 0, 0);
        fence_proxy_async();
    }
    if (warp == 1) {
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

    if (warp == 0 || warp == kVWarp) {
        // ------------------------------------------------------------ producers
        // warp 0: Q once per item and the K ring; warp kVWarp: the V ring.  Both
        // walk the same item and column sequence, so their ring indices agree
        // with the MMA thread's.
        const bool kside = warp == 0;
        if (lane == 0) {
            uint32_t kv_it = 0, q_it = 0;
            bool ok = true;
            for (int k = 0; ok; ++k) {
                const int idx = item_index(k, cta, grid);
                if (idx >= prm.rows) break;
                const int r = prm.work[idx];
                const int beg = prm.row_ptr[r], end = prm.row_ptr[r + 1];
                if (end <= beg) continue;                    // no key block: no Q either
                const int bh = r / nb, i = r % nb;
                if (kside) {
                    if (q_it > 0 && !(ok = mbar_wait<kEvery>(bar(B_QEMPTY), (q_it - 1) & 1, ctl))) break;
                    mbar_expect_tx(bar(B_QFULL), BLK * D * 2);
                    for (int s = 0; s < D / 64; ++s)
                        tma_load_2d(sbase + L::offQ + s * kTileM * 128, &tmQ, s * 64,
                                    (int)(bh * prm.npad + (int64_t)i * BLK), bar(B_QFULL));
                    ++q_it;
                }
                int jn = prm.col_idx[beg];
                for (int jj = beg; jj < end; ++jj) {
                    const int j = jn;
                    if (jj + 1 < end) jn = prm.col_idx[jj + 1];   // next column, one iteration ahead
                    if (!valid_col(j, nb)) {
                        if (kside) record_error(prm.err, BSA_EDEVICE, r);
                        continue;
                    }
                    const int y = (int)(bh * prm.npad + (int64_t)j * BLK);
                    if (kside) {
                        const int st = kv_it % kKStages;
                        const uint32_t use = kv_it / kKStages;
                        if (use > 0 && !(ok = mbar_wait<kEvery>(bar(B_KEMPTY0 + st), (use - 1) & 1, ctl))) break;
                        mbar_expect_tx(bar(B_KFULL0 + st), L::kKV);
                        for (int s = 0; s < D / 64; ++s)
                            tma_load_2d(sbase + L::offK + st * L::kKV + s * BLK * 128, &tmK, s * 64, y,
                                        bar(B_KFULL0 + st));
                    } else {
                        const int st = kv_it % kVStages;
                        const uint32_t use = kv_it / kVStages;
                        if (use > 0 && !(ok = mbar_wait<kEvery>(bar(B_VEMPTY0 + st), (use - 1) & 1, ctl))) break;
                        mbar_expect_tx(bar(B_VFULL0 + st), L::kKV);
                        for (int s = 0; s < D / 64; ++s)
                            tma_load_2d(sbase + L::offV + st * L::kKV + s * BLK * 128, &tmV, s * 64, y,
                                        bar(B_VFULL0 + st));
                    }
                    ++kv_it;
                }
            }
            if (!ok) { ctl->abort = 1; record_error(prm.err, BSA_EDEVICE, -1); }
            // every tile this thread issued lands before the CTA exits (the last
            // load of each stage completes its phase; nothing is issued after it)
            const uint32_t stages = kside ? kKStages : kVStages;
            for (uint32_t st = 0; st < stages; ++st) {
                const uint32_t loads = kv_it > st ? (kv_it - 1 - st) / stages + 1 : 0;
                if (loads > 0) mbar_drain(bar((kside ? B_KFULL0 : B_VFULL0) + st), (loads - 1) & 1);
            }
            if (kside && q_it > 0) mbar_drain(bar(B_QFULL), (q_it - 1) & 1);
        }
    } else if (warp == 1) {
        // ----------------------------------------------------------------- MMA
        if (lane == 0) {
            constexpr uint32_t idesc_qk = instr_desc(BLK, 0);
            constexpr uint32_t idesc_pv = instr_desc(D, 1);
            uint32_t kv_it = 0, q_it = 0, pv_it = 0;
            bool ok = true;
            // O += P V for kv iteration `it`; P sits in TMEM buffer it&1
            auto issue_pv = [&](uint32_t it, bool first) -> bool {
                if (!mbar_wait<kEvery>(bar(B_PFULL), pv_it & 1, ctl)) return false;
                const int st = it % kVStages;
                if (!mbar_wait<kEvery>(bar(B_VFULL0 + st), (it / kVStages) & 1, ctl)) return false;
                fence_after();
                const uint32_t p_tmem = tmem + ((it & 1) ? kColS1 : kColS0);   // P overwrote S(it)
#pragma unroll
                for (int kk = 0; kk < BLK / 16; ++kk) {
                    const uint64_t b = smem_desc(sbase + L::offV + st * L::kKV + kk * 16 * 128, BLK * 128, 1024);
                    mma_ts(tmem + kColO, p_tmem + kk * 8, b, idesc_pv, (first && kk == 0) ? 0u : 1u);
                }
                commit(bar(B_PVDONE));
                commit(bar(B_VEMPTY0 + st));
                ++pv_it;
                return true;
            };
            for (int k = 0; ok; ++k) {
                const int idx = item_index(k, cta, grid);
                if (idx >= prm.rows) break;
                const int r = prm.work[idx];
                const int beg = prm.row_ptr[r], end = prm.row_ptr[r + 1];
                if (end <= beg) continue;
                if (!(ok = mbar_wait<kEvery>(bar(B_QFULL), q_it & 1, ctl))) break;
                ++q_it;
                // Q -> TMEM (16 columns of bf16 per copy), then its shared buffer is free.
                // The previous item's QKs have completed: the last PV issued above waited
                // for that item's last P, which the softmax warps write only after that
                // block's QK result arrived (a copy is not ordered behind earlier MMAs).
                fence_after();
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk)
                    cp_128x256b(tmem + kColQ + kk * 8,
                                   smem_desc(sbase + L::offQ + (kk / 4) * kTileM * 128 + (kk % 4) * 32, 16, 1024));
                commit(bar(B_QEMPTY));
                int local = 0;
                int jn = prm.col_idx[beg];
                for (int jj = beg; jj < end && ok; ++jj) {
                    const int j = jn;
                    if (jj + 1 < end) jn = prm.col_idx[jj + 1];   // next column, one iteration ahead
                    if (!valid_col(j, nb)) continue;
                    const int st = kv_it % kKStages;
                    // S buffer kv_it&1 is free: the softmax warps read S(kv_it-2) before the
                    // P_FULL arrival this thread waited on for PV(kv_it-2), and that PV, which
                    // read P from the same columns, was issued earlier by this thread.
                    if (!(ok = mbar_wait<kEvery>(bar(B_KFULL0 + st), (kv_it / kKStages) & 1, ctl))) break;
                    fence_after();
                    const uint32_t d_s = tmem + ((kv_it & 1) ? kColS1 : kColS0);
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint64_t b = smem_desc(sbase + L::offK + st * L::kKV + (kk / 4) * BLK * 128 + (kk % 4) * 32, 16, 1024);
                        mma_ts(d_s, tmem + kColQ + kk * 8, b, idesc_qk, kk > 0 ? 1u : 0u);
                    }
                    commit(bar(B_SFULL0 + (kv_it & 1)));
                    commit(bar(B_KEMPTY0 + st));
                    if (local > 0 && !(ok = issue_pv(kv_it - 1, local == 1))) break;
                    ++kv_it;
                    ++local;
                }
                if (!ok) break;
                if (local > 0 && !(ok = issue_pv(kv_it - 1, local == 1))) break;
            }
            if (!ok) {
                ctl->abort = 1;
                record_error(prm.err, BSA_EDEVICE, -2);
            }
            // drain: everything this thread issued completes before TMEM is freed
            commit(bar(B_DRAIN));
            mbar_drain(bar(B_DRAIN), 0);
        }
    } else {
        // ------------------------------------------------------------- softmax
        const int quad = warp & 3;                       // TMEM lane quadrant
        const int half = (warp - 2) >> 2;                // which half of the key / output columns
        const int row = 32 * quad + lane;                // TMEM lane == query row in tile
        const uint32_t lane_base = (uint32_t)(32 * quad) << 16;
        uint32_t kv_it = 0, pv_it = 0, items = 0, pairs = 0;
        bool ok = true;
        for (int k = 0; ok; ++k) {
            const int idx = item_index(k, cta, grid);
            if (idx >= prm.rows) break;
            const int r = prm.work[idx];
            const int beg = prm.row_ptr[r], end = prm.row_ptr[r + 1];
            const int bh = r / nb, i = r % nb;
            const int b = bh / prm.H, h = bh % prm.H;
            const int n_tok = i * BLK + row;             // reordered position of this row
            const bool row_real = row < BLK && n_tok < prm.N;
            __nv_bfloat16* dst = prm.o + (((int64_t)b * prm.N + (row_real ? prm.perm[n_tok] : 0)) * prm.H + h) * D +
                                 half * OC;
            float m_use = 0.f, l = 0.f;
            int local = 0;
            int jn = end > beg ? prm.col_idx[beg] : 0;
            for (int jj = beg; jj < end && ok; ++jj) {
                const int j = jn;
                if (jj + 1 < end) jn = prm.col_idx[jj + 1];   // next column, one iteration ahead
                if (!valid_col(j, nb)) continue;
                const int sb = kv_it & 1;
                const uint32_t s_col = sb ? kColS1 : kColS0;
                if (!(ok = warp_wait<kEvery>(bar(B_SFULL0 + sb), (kv_it >> 1) & 1, ctl))) break;
                fence_after();
                // padding keys of a ragged last block
                const int valid_keys = prm.N - j * BLK;
                const bool ragged = valid_keys < BLK;
                uint32_t sv[HC];                          // this warp's half of the S row
#pragma unroll
                for (int c = 0; c < HC / 32; ++c) tmem_ld32(tmem + lane_base + s_col + half * HC + c * 32, sv + 32 * c);
                tmem_wait_ld();
                if (ragged) {
#pragma unroll
                    for (int c = 0; c < HC; ++c)
                        if (half * HC + c >= valid_keys) sv[c] = __float_as_uint(-INFINITY);
                }
                // the two half-row maxima meet in shared memory (slots alternate with
                // the kv parity; the pair mbarrier completes once per block)
                const float lmax = row_max<HC>(sv, -INFINITY);
                float* xs = xchg + sb * 2 * kTileM;
                xs[half * kTileM + row] = lmax;
                mbar_arrive(bar(B_PAIR0 + quad));
                if (!(ok = warp_wait<kEvery>(bar(B_PAIR0 + quad), pairs & 1, ctl))) break;
                ++pairs;
                const float mx = fmaxf(lmax, xs[(1 - half) * kTileM + row]) * prm.scale_log2;
                float alpha = 1.f;
                bool rescale = false;
                if (local == 0) {
                    m_use = mx;
                } else if (mx > m_use + 8.f) {
                    alpha = ex2_mufu(m_use - mx);
                    m_use = mx;
                    rescale = true;
                }
                uint32_t pk[HC / 2];
                const float rowsum = ragged ? softmax_half<HC, true>(sv, prm.scale_log2, -m_use, pk)
                                            : softmax_half<HC, false>(sv, prm.scale_log2, -m_use, pk);
                l = l * alpha + rowsum;
                // P_j (bf16 pairs) over the first half of S_j's columns: both warps of the
                // pair read their S halves before the exchange above.
                const uint32_t p_addr = tmem + lane_base + s_col + half * (HC / 2);
                if constexpr (HC / 2 == 32) {
                    tmem_st32(p_addr, pk);
                } else {
                    tmem_st16(p_addr, pk);
                }
                // the previous PV must be done before O is rescaled; waiting on it every
                // block keeps at most one PV completion outstanding for this warp
                if (local > 0) {
                    if (!(ok = warp_wait<kEvery>(bar(B_PVDONE), pv_it & 1, ctl))) break;
                    ++pv_it;
                    fence_after();
                    if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
                        for (int c = 0; c < OC / 32; ++c) {
                            uint32_t o[32];
                            tmem_ld32(tmem + lane_base + kColO + half * OC + c * 32, o);
                            tmem_wait_ld();
#pragma unroll
                            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                            tmem_st32(tmem + lane_base + kColO + half * OC + c * 32, o);
                        }
                    }
                }
                tmem_wait_st();
                fence_before();
                mbar_arrive(bar(B_PFULL));
                ++kv_it;
                ++local;
            }
            if (!ok) break;
            if (local == 0) {                            // no (valid) key block: zeros
                if (row_real)
                    for (int c = 0; c < OC / 8; ++c) reinterpret_cast<uint4*>(dst)[c] = make_uint4(0, 0, 0, 0);
                continue;
            }
            // epilogue: last PV of the item; the two partial row sums meet in shared
            // memory (slots alternate by item; a bounded mbarrier pairs the two warps)
            if (!(ok = warp_wait<kEvery>(bar(B_PVDONE), pv_it & 1, ctl))) break;
            ++pv_it;
            fence_after();
            float* ls = xchg + 4 * kTileM + (items & 1) * 2 * kTileM;
            ls[half * kTileM + row] = l;
            mbar_arrive(bar(B_PAIR0 + quad));
            if (!(ok = warp_wait<kEvery>(bar(B_PAIR0 + quad), pairs & 1, ctl))) break;
            ++pairs;
            ++items;
            const float inv = 1.f / (l + ls[(1 - half) * kTileM + row]);
#pragma unroll
            for (int c = 0; c < OC / 32; ++c) {
                uint32_t o[32];
                tmem_ld32(tmem + lane_base + kColO + half * OC + c * 32, o);
                tmem_wait_ld();
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
        }
        if (!ok) { ctl->abort = 1; record_error(prm.err, BSA_EDEVICE, -3); }
        tmem_wait_st();                                  // no TMEM access of this warp outlives the loop
        tmem_wait_ld();
    }

    fence_before();
    __syncthreads();
    fence_after();
    if (warp == 1) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
    }
}

// ----------------------------------------------------------------- host side
template <int D, int BLK, uint32_t kEvery>
cudaError_t launch_t(const bsa_plan& p, const void* qp, const void* kp, const void* vp, const Params& prm,
                     cudaStream_t s) {
    using L = Smem<D, BLK>;
    const int64_t rows_total = (int64_t)p.B * p.H * p.nb * p.block;
    CUtensorMap mq, mk, mv;
    if (!make_map(&mq, qp, rows_total, D, BLK) || !make_map(&mk, kp, rows_total, D, BLK) ||
        !make_map(&mv, vp, rows_total, D, BLK))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(k_attn_tc<D, BLK, kEvery>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         L::kAlloc);
    if (e != cudaSuccess) return e;
    const int grid = (int)std::min<int64_t>(p.num_sms, p.rows);
    k_attn_tc<D, BLK, kEvery><<<grid, kThreads, L::kAlloc, s>>>(mq, mk, mv, prm);
    return cudaGetLastError();
}

// a wait limit below a millisecond: the variant that checks it at every probe
template <int D, int BLK>
cudaError_t launch(const bsa_plan& p, const void* qp, const void* kp, const void* vp, const Params& prm,
                   cudaStream_t s) {
    if (prm.wait_ns < 1000000ull) return launch_t<D, BLK, 0>(p, qp, kp, vp, prm, s);
    return launch_t<D, BLK, 1023>(p, qp, kp, vp, prm, s);
}

}  // namespace

cudaError_t launch_attn_tc(const bsa_plan& p, const void* qp, const void* kp, const void* vp,
                           const int32_t* row_ptr, const int32_t* col_idx, const int32_t* work,
                           int32_t* counter, void* o, cudaStream_t s) {
    (void)counter;
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
    prm.wait_ns = p.wait_ns;
    if (p.d == 128 && p.block == 128) return launch<128, 128>(p, qp, kp, vp, prm, s);
    if (p.d == 128 && p.block == 64) return launch<128, 64>(p, qp, kp, vp, prm, s);
    if (p.d == 64 && p.block == 128) return launch<64, 128>(p, qp, kp, vp, prm, s);
    return launch<64, 64>(p, qp, kp, vp, prm, s);
}


}  // namespace bsa
