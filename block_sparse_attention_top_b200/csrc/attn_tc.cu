// Persistent block-sparse attention on the 5th-generation tensor cores
// (FVAttn review, section 3 "Block-Sparse Attention Execution": attention
// computed only over the retained key blocks, outputs restored to token order).
//
// One CTA per SM walks a static zig-zag share of the heaviest-first work list
// (one item = one 128-row query tile of one head).  Per item and retained key
// block j, with S and O living in tensor memory (TMEM):
//
//   warp 0 (1 thread)   TMA: Q tile once per item; K_j, V_j into 2-stage rings
//   warp 1 (1 thread)   tcgen05.mma: S[j%2] = Q K_j^T   (M=128, N=block, K=d)
//                                    O     += P_j V_j   (M=128, N=d,     K=block)
//   warps 2..5          softmax: thread = query row = TMEM lane; reads S[j%2]
//                       (tcgen05.ld), online softmax in the log2 domain, writes
//                       P_j (bf16) into a 128B-swizzled shared tile, rescales the
//                       O row in TMEM only when its running max grows by more
//                       than 2^8; epilogue: O / l, bf16, stored at the token's
//                       raster position (the inverse Hilbert permutation is
//                       fused into this store).
//
// S is double-buffered, so QK^T of block j+1 and PV of block j-1 run on the
// tensor pipe while the softmax warps work on block j.
//
// Every wait on an mbarrier is bounded (about 4 s of %globaltimer); on expiry
// the CTA records BSA_EDEVICE, raises a shared abort flag that stops the other
// roles, drains its own tensor-core work and frees TMEM before returning.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "bsa_internal.cuh"

namespace bsa {
namespace {

constexpr int kThreads = 192;           // 6 warps
constexpr int kTileM = 128;             // query rows per tile (TMEM lanes)
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO = 256;
constexpr unsigned long long kTimeoutNs = 4000000000ull;

// ---------------------------------------------------------------- PTX helpers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ unsigned long long globaltimer() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
// Bounded wait: false if the abort flag is raised or the time limit passes.
__device__ __noinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = globaltimer();
    for (uint32_t n = 1;; ++n) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((n & 63u) == 0) {
            if (*abort_flag) return false;
            if (globaltimer() - t0 > kTimeoutNs) return false;
        }
    }
}
// Warp-uniform bounded wait (every lane polls; all lanes agree on the outcome).
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag));
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}
__device__ __forceinline__ void fence_proxy_async() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}
// D[tmem] (+)= A[smem desc] * B[smem desc]
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"
        ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
          "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]),
          "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]),
          "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Shared-memory matrix descriptor, 128-byte swizzle, sm_100 format (version 1).
// lbo / sbo in bytes.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}
// Instruction descriptor, kind::f16: bf16 A and B, fp32 accumulator, M = 128.
__host__ __device__ constexpr uint32_t instr_desc(int n, int b_mn_major) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)b_mn_major << 16) | ((uint32_t)(n >> 3) << 17) |
           ((uint32_t)(kTileM >> 4) << 24);
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// ------------------------------------------------------------- shared layout
template <int D, int BLK>
struct Smem {
    static constexpr int kQ = kTileM * D * 2;       // Q tile, D/64 column slabs of 128 rows
    static constexpr int kKV = BLK * D * 2;         // one K or V tile
    static constexpr int kP = kTileM * BLK * 2;     // P tile, BLK/64 slabs of 128 rows
    static constexpr int offQ = 0;
    static constexpr int offK = offQ + kQ;
    static constexpr int offV = offK + 2 * kKV;
    static constexpr int offP = offV + 2 * kKV;
    static constexpr int offBar = offP + kP;
    static constexpr int kBars = 17;
    static constexpr int offMisc = offBar + kBars * 8;
    static constexpr int kBytes = offMisc + 64;
    static constexpr int kAlloc = kBytes + 1024;   // room to align the base to 1024 B
};
// barrier slots
enum { B_QFULL = 0, B_QEMPTY, B_KFULL0, B_KFULL1, B_KEMPTY0, B_KEMPTY1, B_VFULL0, B_VFULL1, B_VEMPTY0,
       B_VEMPTY1, B_SFULL0, B_SFULL1, B_SEMPTY0, B_SEMPTY1, B_PFULL, B_PVDONE, B_DRAIN, B_COUNT };

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
};

// Work item sequence of this CTA: zig-zag over the heaviest-first list.
__device__ __forceinline__ int item_index(int k, int cta, int grid) {
    return k * grid + ((k & 1) ? (grid - 1 - cta) : cta);
}

__device__ __forceinline__ bool valid_col(int j, int nb) { return j >= 0 && j < nb; }

template <int D, int BLK>
__global__ void __launch_bounds__(kThreads, 1)
k_attn_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
          const __grid_constant__ CUtensorMap tmV, const Params prm) {
    using L = Smem<D, BLK>;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    const uint32_t bar0 = sbase + L::offBar;
    auto bar = [&](int i) { return bar0 + 8u * (uint32_t)i; };
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::offMisc);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::offMisc + 8);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

    if (threadIdx.x == 0) {
        *abort_flag = 0;
        for (int i = 0; i < B_COUNT; ++i)
            mbar_init(bar(i), (i == B_SEMPTY0 || i == B_SEMPTY1 || i == B_PFULL) ? 128u : 1u);
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
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    const int grid = gridDim.x, cta = blockIdx.x;
    const int nb = prm.nb;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            uint32_t kv_it = 0, q_it = 0;
            bool ok = true;
            for (int k = 0; ok; ++k) {
                const int idx = item_index(k, cta, grid);
                if (idx >= prm.rows) break;
                const int r = prm.work[idx];
                const int beg = prm.row_ptr[r], end = prm.row_ptr[r + 1];
                int nvalid = 0;
                for (int jj = beg; jj < end; ++jj) nvalid += valid_col(prm.col_idx[jj], nb);
                if (nvalid == 0) continue;
                const int bh = r / nb, i = r % nb;
                if (q_it > 0 && !(ok = mbar_wait(bar(B_QEMPTY), (q_it - 1) & 1, abort_flag))) break;
                mbar_expect_tx(bar(B_QFULL), BLK * D * 2);
                for (int s = 0; s < D / 64; ++s)
                    tma_load_2d(sbase + L::offQ + s * kTileM * 128, &tmQ, s * 64,
                                (int)(bh * prm.npad + (int64_t)i * BLK), bar(B_QFULL));
                ++q_it;
                for (int jj = beg; jj < end; ++jj) {
                    const int j = prm.col_idx[jj];
                    if (!valid_col(j, nb)) {
                        record_error(prm.err, BSA_EDEVICE, r);
                        continue;
                    }
                    const int st = kv_it & 1;
                    const uint32_t ph = ((kv_it >> 1) & 1) ^ 1;
                    const int y = (int)(bh * prm.npad + (int64_t)j * BLK);
                    if (kv_it >= 2 && !(ok = mbar_wait(bar(B_KEMPTY0 + st), ph, abort_flag))) break;
                    mbar_expect_tx(bar(B_KFULL0 + st), L::kKV);
                    for (int s = 0; s < D / 64; ++s)
                        tma_load_2d(sbase + L::offK + st * L::kKV + s * BLK * 128, &tmK, s * 64, y, bar(B_KFULL0 + st));
                    if (kv_it >= 2 && !(ok = mbar_wait(bar(B_VEMPTY0 + st), ph, abort_flag))) break;
                    mbar_expect_tx(bar(B_VFULL0 + st), L::kKV);
                    for (int s = 0; s < D / 64; ++s)
                        tma_load_2d(sbase + L::offV + st * L::kKV + s * BLK * 128, &tmV, s * 64, y, bar(B_VFULL0 + st));
                    ++kv_it;
                }
            }
            if (!ok) { *abort_flag = 1; record_error(prm.err, BSA_EDEVICE, -1); }
        }
    } else if (warp == 1) {
        // ----------------------------------------------------------------- MMA
        if (lane == 0) {
            constexpr uint32_t idesc_qk = instr_desc(BLK, 0);
            constexpr uint32_t idesc_pv = instr_desc(D, 1);
            uint32_t kv_it = 0, q_it = 0, pv_it = 0;
            bool ok = true;
            // PV of iteration `it` (stage it&1) for the item's local block `first`
            auto issue_pv = [&](uint32_t it, bool first) -> bool {
                if (!mbar_wait(bar(B_PFULL), pv_it & 1, abort_flag)) return false;
                const int st = it & 1;
                if (!mbar_wait(bar(B_VFULL0 + st), (it >> 1) & 1, abort_flag)) return false;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < BLK / 16; ++kk) {
                    const uint64_t a = smem_desc(sbase + L::offP + (kk / 4) * kTileM * 128 + (kk % 4) * 32, 16, 1024);
                    const uint64_t b = smem_desc(sbase + L::offV + st * L::kKV + kk * 16 * 128, BLK * 128, 1024);
                    tc_mma(tmem + kColO, a, b, idesc_pv, (first && kk == 0) ? 0u : 1u);
                }
                tc_commit(bar(B_PVDONE));
                tc_commit(bar(B_VEMPTY0 + st));
                ++pv_it;
                return true;
            };
            for (int k = 0; ok; ++k) {
                const int idx = item_index(k, cta, grid);
                if (idx >= prm.rows) break;
                const int r = prm.work[idx];
                const int beg = prm.row_ptr[r], end = prm.row_ptr[r + 1];
                int nvalid = 0;
                for (int jj = beg; jj < end; ++jj) nvalid += valid_col(prm.col_idx[jj], nb);
                if (nvalid == 0) continue;
                if (!(ok = mbar_wait(bar(B_QFULL), q_it & 1, abort_flag))) break;
                ++q_it;
                int local = 0;
                for (int jj = beg; jj < end && ok; ++jj) {
                    if (!valid_col(prm.col_idx[jj], nb)) continue;
                    const int st = kv_it & 1;
                    const int sb = kv_it & 1;     // S buffer follows the kv iteration
                    if (!(ok = mbar_wait(bar(B_KFULL0 + st), (kv_it >> 1) & 1, abort_flag))) break;
                    if (kv_it >= 2 && !(ok = mbar_wait(bar(B_SEMPTY0 + sb), ((kv_it >> 1) & 1) ^ 1, abort_flag))) break;
                    tc_fence_after();
                    const uint32_t d_s = tmem + (sb ? kColS1 : kColS0);
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint64_t a = smem_desc(sbase + L::offQ + (kk / 4) * kTileM * 128 + (kk % 4) * 32, 16, 1024);
                        const uint64_t b = smem_desc(sbase + L::offK + st * L::kKV + (kk / 4) * BLK * 128 + (kk % 4) * 32, 16, 1024);
                        tc_mma(d_s, a, b, idesc_qk, kk > 0 ? 1u : 0u);
                    }
                    tc_commit(bar(B_SFULL0 + sb));
                    tc_commit(bar(B_KEMPTY0 + st));
                    if (local == nvalid - 1) tc_commit(bar(B_QEMPTY));
                    if (local > 0 && !(ok = issue_pv(kv_it - 1, local == 1))) break;
                    ++kv_it;
                    ++local;
                }
                if (ok && !(ok = issue_pv(kv_it - 1, nvalid == 1))) break;
            }
            if (!ok) {
                *abort_flag = 1;
                record_error(prm.err, BSA_EDEVICE, -2);
            }
            // drain: everything this thread issued completes before TMEM is freed
            tc_commit(bar(B_DRAIN));
            volatile int no_abort = 0;
            mbar_wait(bar(B_DRAIN), 0, &no_abort);
        }
    } else {
        // ------------------------------------------------------------- softmax
        const int row = 32 * (warp & 3) + lane;          // TMEM lane == query row in tile
        const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
        uint32_t kv_it = 0, pv_it = 0;
        bool ok = true;
        for (int k = 0; ok; ++k) {
            const int idx = item_index(k, cta, grid);
            if (idx >= prm.rows) break;
            const int r = prm.work[idx];
            const int beg = prm.row_ptr[r], end = prm.row_ptr[r + 1];
            int nvalid = 0;
            for (int jj = beg; jj < end; ++jj) nvalid += valid_col(prm.col_idx[jj], nb);
            const int bh = r / nb, i = r % nb;
            const int b = bh / prm.H, h = bh % prm.H;
            const int n_tok = i * BLK + row;             // reordered position of this row
            const bool row_real = row < BLK && n_tok < prm.N;
            if (nvalid == 0) {
                if (row_real) {
                    uint4* dst = reinterpret_cast<uint4*>(prm.o + (((int64_t)b * prm.N + prm.perm[n_tok]) * prm.H + h) * D);
                    for (int c = 0; c < D / 8; ++c) dst[c] = make_uint4(0, 0, 0, 0);
                }
                continue;
            }
            float m_use = 0.f, l = 0.f;
            int local = 0;
            for (int jj = beg; jj < end && ok; ++jj) {
                const int j = prm.col_idx[jj];
                if (!valid_col(j, nb)) continue;
                const int sb = kv_it & 1;
                if (!(ok = warp_wait(bar(B_SFULL0 + sb), (kv_it >> 1) & 1, abort_flag))) break;
                tc_fence_after();
                float s[BLK];
                {
                    uint32_t raw[32];
#pragma unroll
                    for (int c = 0; c < BLK / 32; ++c) {
                        tmem_ld32(tmem + lane_base + (sb ? kColS1 : kColS0) + c * 32, raw);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e) s[c * 32 + e] = __uint_as_float(raw[e]);
                    }
                }
                tc_fence_before();
                mbar_arrive(bar(B_SEMPTY0 + sb));
                // mask the padding keys of a ragged last block
                const int valid_keys = min(BLK, prm.N - j * BLK);
                float mx = -INFINITY;
#pragma unroll
                for (int c = 0; c < BLK; ++c) {
                    s[c] = c < valid_keys ? s[c] * prm.scale_log2 : -INFINITY;
                    mx = fmaxf(mx, s[c]);
                }
                float alpha = 1.f;
                bool rescale = false;
                if (local == 0) {
                    m_use = mx;
                } else if (mx > m_use + 8.f) {
                    alpha = exp2f(m_use - mx);
                    m_use = mx;
                    rescale = true;
                }
                float rowsum = 0.f;
                uint32_t packed[BLK / 2];
#pragma unroll
                for (int c = 0; c < BLK; c += 2) {
                    const float p0 = exp2f(s[c] - m_use);
                    const float p1 = exp2f(s[c + 1] - m_use);
                    rowsum += p0 + p1;
                    packed[c / 2] = pack_bf16(p0, p1);
                }
                l = l * alpha + rowsum;
                // the previous PV must be done before P is overwritten and O is touched
                if (local > 0) {
                    if (!(ok = warp_wait(bar(B_PVDONE), pv_it & 1, abort_flag))) break;
                    ++pv_it;
                    tc_fence_after();
                }
                // P row -> swizzled smem slab(s): 16-byte chunk u of row `row` lands at
                // chunk u ^ (row % 8) inside the row's 128-byte line
                unsigned char* prow = smem + L::offP + (row / 8) * 1024 + (row % 8) * 128;
#pragma unroll
                for (int u = 0; u < BLK / 8; ++u) {
                    const int slab = u / 8, cu = u % 8;
                    uint4 v = make_uint4(packed[4 * u], packed[4 * u + 1], packed[4 * u + 2], packed[4 * u + 3]);
                    *reinterpret_cast<uint4*>(prow + slab * kTileM * 128 + ((cu ^ (row % 8)) * 16)) = v;
                }
                if (__any_sync(0xffffffffu, rescale)) {
                    const float a = rescale ? alpha : 1.f;
#pragma unroll
                    for (int c = 0; c < D / 32; ++c) {
                        uint32_t o[32];
                        tmem_ld32(tmem + lane_base + kColO + c * 32, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * a);
                        tmem_st32(tmem + lane_base + kColO + c * 32, o);
                    }
                    tmem_wait_st();
                }
                fence_proxy_async();
                tc_fence_before();
                mbar_arrive(bar(B_PFULL));
                ++kv_it;
                ++local;
            }
            if (!ok) break;
            // epilogue: last PV of the item, then O / l to the token's raster position
            if (!(ok = warp_wait(bar(B_PVDONE), pv_it & 1, abort_flag))) break;
            ++pv_it;
            tc_fence_after();
            const float inv = 1.f / l;
            __nv_bfloat16* dst = prm.o + (((int64_t)b * prm.N + (row_real ? prm.perm[n_tok] : 0)) * prm.H + h) * D;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t o[32];
                tmem_ld32(tmem + lane_base + kColO + c * 32, o);
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
            tc_fence_before();
        }
        if (!ok) { *abort_flag = 1; record_error(prm.err, BSA_EDEVICE, -3); }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
    }
}

// ----------------------------------------------------------------- host side
PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// [rows, d] bf16 row-major, box = [box_rows, 64] with 128-byte swizzle
bool make_map(CUtensorMap* m, const void* base, int64_t rows, int d, int box_rows) {
    auto enc = get_encode();
    if (!enc) return false;
    cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)d * 2};
    cuuint32_t box[2] = {64u, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1u, 1u};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, int BLK>
cudaError_t launch(const bsa_plan& p, const void* qp, const void* kp, const void* vp, const Params& prm,
                   cudaStream_t s) {
    using L = Smem<D, BLK>;
    const int64_t rows_total = (int64_t)p.B * p.H * p.nb * p.block;
    CUtensorMap mq, mk, mv;
    if (!make_map(&mq, qp, rows_total, D, BLK) || !make_map(&mk, kp, rows_total, D, BLK) ||
        !make_map(&mv, vp, rows_total, D, BLK))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(k_attn_tc<D, BLK>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
    if (e != cudaSuccess) return e;
    const int grid = (int)std::min<int64_t>(p.num_sms, p.rows);
    k_attn_tc<D, BLK><<<grid, kThreads, L::kAlloc, s>>>(mq, mk, mv, prm);
    return cudaGetLastError();
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
    if (p.d == 128 && p.block == 128) return launch<128, 128>(p, qp, kp, vp, prm, s);
    if (p.d == 128 && p.block == 64) return launch<128, 64>(p, qp, kp, vp, prm, s);
    if (p.d == 64 && p.block == 128) return launch<64, 128>(p, qp, kp, vp, prm, s);
    return launch<64, 64>(p, qp, kp, vp, prm, s);
}

}  // namespace bsa
