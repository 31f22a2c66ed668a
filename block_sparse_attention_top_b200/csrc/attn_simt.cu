// Slow CUDA-core cross-check of the block-sparse attention (FVAttn review,
// section 3 "Block-Sparse Attention Execution"): one warp per query token,
// each lane owning d/32 dimensions, keys visited one at a time with an fp32
// online softmax.  Same inputs (reordered tiles + CSR) and same output
// contract as the tensor-core kernel; used by the tests, never by the bench.
#include <cuda_bf16.h>

#include "bsa_internal.cuh"

namespace bsa {
namespace {

constexpr int kWarps = 8;

template <int D>
__global__ void __launch_bounds__(kWarps * 32)
k_attn_simt(const __nv_bfloat16* __restrict__ qp, const __nv_bfloat16* __restrict__ kp,
            const __nv_bfloat16* __restrict__ vp, const int32_t* __restrict__ row_ptr,
            const int32_t* __restrict__ col_idx, __nv_bfloat16* __restrict__ o,
            const int32_t* __restrict__ perm, int N, int H, int nb, int block, int32_t* err) {
    constexpr int DPL = D / 32;
    const int groups = block / kWarps;
    const int64_t r = blockIdx.x / groups;
    const int tok = (blockIdx.x % groups) * kWarps + threadIdx.x / 32;
    const int lane = threadIdx.x % 32;
    const int64_t bh = r / nb;
    const int i = (int)(r % nb);
    const int n = i * block + tok;
    if (n >= N) return;
    const int64_t npad = (int64_t)nb * block;
    const __nv_bfloat16* qrow = qp + (bh * npad + n) * D + lane * DPL;
    float q[DPL], acc[DPL];
#pragma unroll
    for (int e = 0; e < DPL; ++e) { q[e] = __bfloat162float(qrow[e]); acc[e] = 0.f; }
    const float scale_log2 = 1.4426950408889634f / sqrtf((float)D);
    float m = -INFINITY, l = 0.f;
    const int beg = row_ptr[r], end = row_ptr[r + 1];
    for (int jj = beg; jj < end; ++jj) {
        const int j = col_idx[jj];
        if (j < 0 || j >= nb) {
            if (lane == 0) record_error(err, BSA_EDEVICE, (int)r);
            continue;
        }
        const int t_end = min(N, (j + 1) * block);
        for (int t = j * block; t < t_end; ++t) {
            const __nv_bfloat16* krow = kp + (bh * npad + t) * D + lane * DPL;
            const __nv_bfloat16* vrow = vp + (bh * npad + t) * D + lane * DPL;
            float s = 0.f;
#pragma unroll
            for (int e = 0; e < DPL; ++e) s = fmaf(q[e], __bfloat162float(krow[e]), s);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
            s *= scale_log2;
            const float m_new = fmaxf(m, s);
            const float corr = exp2f(m - m_new);
            const float pw = exp2f(s - m_new);
            l = l * corr + pw;
#pragma unroll
            for (int e = 0; e < DPL; ++e) acc[e] = fmaf(pw, __bfloat162float(vrow[e]), acc[e] * corr);
            m = m_new;
        }
    }
    const float inv = l > 0.f ? 1.f / l : 0.f;
    const int b = (int)(bh / H), h = (int)(bh % H);
    __nv_bfloat16* orow = o + (((int64_t)b * N + perm[n]) * H + h) * D + lane * DPL;
#pragma unroll
    for (int e = 0; e < DPL; ++e) orow[e] = __float2bfloat16(acc[e] * inv);
}

}  // namespace

cudaError_t launch_attn_simt(const bsa_plan& p, const void* qp, const void* kp, const void* vp,
                             const int32_t* row_ptr, const int32_t* col_idx, const int32_t* work,
                             void* o, cudaStream_t s) {
    (void)work;
    const unsigned grid = (unsigned)(p.rows * (p.block / kWarps));
    if (p.d == 128)
        k_attn_simt<128><<<grid, kWarps * 32, 0, s>>>((const __nv_bfloat16*)qp, (const __nv_bfloat16*)kp,
                                                      (const __nv_bfloat16*)vp, row_ptr, col_idx,
                                                      (__nv_bfloat16*)o, p.d_perm, (int)p.N, p.H, (int)p.nb,
                                                      p.block, p.d_err);
    else
        k_attn_simt<64><<<grid, kWarps * 32, 0, s>>>((const __nv_bfloat16*)qp, (const __nv_bfloat16*)kp,
                                                     (const __nv_bfloat16*)vp, row_ptr, col_idx,
                                                     (__nv_bfloat16*)o, p.d_perm, (int)p.N, p.H, (int)p.nb,
                                                     p.block, p.d_err);
    return cudaGetLastError();
}

}  // namespace bsa
