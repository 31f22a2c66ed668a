// FP8 (e4m3) V for the P.V product (FVAttn review, section 3 "Block-Sparse
// Attention Execution" and section 3.4: V is quantized before attention; the
// format is not stated).  Per head and channel c, sigma_c = amax over the N
// tokens of |V[:, c]| / 448; V[:, c] / sigma_c is rounded to e4m3 (nearest,
// ties to even, saturating) and stored transposed, one [d x 128] byte tile per
// (head, key block) in the reordered token order, so that the P.V MMA reads V
// K-major like every other operand.  Padding tokens of the last block are 0.
//
//   k_vamax    amax |V| per (batch, head, channel): bf16 bit patterns of
//              non-negative values order like unsigned integers, so a plain
//              atomicMax on the 16-bit pattern widened to 32 bits finds it
//   k_quant_vt one CTA per (head, key block): gather 128 rows through the
//              token order into shared memory, scale, round, write d rows of
//              128 bytes
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "bsa_internal.cuh"

namespace bsa {
namespace {

constexpr int kAmaxThreads = 256;

// grid: (ceil(chunks / 256), token slices, B); each thread owns one 16-byte
// chunk (8 channels) of the H*d row and strides over the tokens of its slice.
__global__ void __launch_bounds__(kAmaxThreads)
k_vamax(const uint4* __restrict__ v, int N, int chunks, uint32_t* __restrict__ amax_bits) {
    const int c = blockIdx.x * blockDim.x + threadIdx.x;
    if (c >= chunks) return;
    const int b = blockIdx.z;
    uint32_t m[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    for (int n = blockIdx.y; n < N; n += gridDim.y) {
        const uint4 u = __ldg(v + ((size_t)b * N + n) * chunks + c);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            m[2 * e] = max(m[2 * e], w[e] & 0x7FFFu);
            m[2 * e + 1] = max(m[2 * e + 1], (w[e] >> 16) & 0x7FFFu);
        }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e)
        if (m[e]) atomicMax(amax_bits + ((size_t)b * chunks + c) * 8 + e, m[e]);
}

// sigma_c = amax / 448 (1 for an all-zero channel), in place of the amax bits
__global__ void k_sigma(uint32_t* __restrict__ amax_bits, int64_t n) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    const float a = __uint_as_float(amax_bits[i] << 16);
    reinterpret_cast<float*>(amax_bits)[i] = a > 0.f ? a / 448.f : 1.f;
}

template <int D>
__global__ void __launch_bounds__(256)
k_quant_vt(const __nv_bfloat16* __restrict__ v, const int32_t* __restrict__ perm, const float* __restrict__ sigma,
           int N, int H, int nb, uint8_t* __restrict__ vt) {
    constexpr int kRows = 128;                   // key tokens per block
    constexpr int kPad = 8;                      // bf16 elements of row padding (bank spread)
    __shared__ __align__(16) __nv_bfloat16 tile[kRows][D + kPad];
    __shared__ float inv[D];
    const int j = blockIdx.x;
    const int bh = blockIdx.y;
    const int b = bh / H, h = bh % H;
    for (int c = threadIdx.x; c < D; c += blockDim.x) inv[c] = 1.f / sigma[(size_t)bh * D + c];
    constexpr int kChunks = D / 8;               // 16-byte chunks per token row
    for (int e = threadIdx.x; e < kRows * kChunks; e += blockDim.x) {
        const int r = e / kChunks, ch = e % kChunks;
        const int n = j * kRows + r;
        uint4 u = make_uint4(0, 0, 0, 0);
        if (n < N) u = __ldg(reinterpret_cast<const uint4*>(v + (((size_t)b * N + perm[n]) * H + h) * D) + ch);
        *reinterpret_cast<uint4*>(&tile[r][ch * 8]) = u;
    }
    __syncthreads();
    // output: row c of the tile holds keys 0..127 of channel c; 16 keys per thread-chunk
    uint8_t* out = vt + ((size_t)bh * nb + j) * D * kRows;
    for (int e = threadIdx.x; e < D * (kRows / 16); e += blockDim.x) {
        const int c = e / (kRows / 16), kc = e % (kRows / 16);
        const float s = inv[c];
        uint32_t w[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int k0 = kc * 16 + q * 4;
            const __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(
                make_float2(__bfloat162float(tile[k0][c]) * s, __bfloat162float(tile[k0 + 1][c]) * s),
                __NV_SATFINITE, __NV_E4M3);
            const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(
                make_float2(__bfloat162float(tile[k0 + 2][c]) * s, __bfloat162float(tile[k0 + 3][c]) * s),
                __NV_SATFINITE, __NV_E4M3);
            w[q] = (uint32_t)lo | ((uint32_t)hi << 16);
        }
        *reinterpret_cast<uint4*>(out + (size_t)c * kRows + kc * 16) = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

}  // namespace

cudaError_t launch_quant_v(const bsa_plan& p, const void* v, float* sigma, void* vt, cudaStream_t s) {
    const int chunks = p.H * p.d / 8;
    const int64_t n_sigma = (int64_t)p.B * p.H * p.d;
    cudaError_t e = cudaMemsetAsync(sigma, 0, (size_t)n_sigma * sizeof(float), s);
    if (e != cudaSuccess) return e;
    const int slices = (int)std::min<int64_t>(p.N, 4 * (int64_t)p.num_sms);
    dim3 g1((unsigned)((chunks + kAmaxThreads - 1) / kAmaxThreads), (unsigned)slices, (unsigned)p.B);
    k_vamax<<<g1, kAmaxThreads, 0, s>>>((const uint4*)v, (int)p.N, chunks, reinterpret_cast<uint32_t*>(sigma));
    k_sigma<<<(unsigned)((n_sigma + 255) / 256), 256, 0, s>>>(reinterpret_cast<uint32_t*>(sigma), n_sigma);
    dim3 g2((unsigned)p.nb, (unsigned)(p.B * p.H));
    if (p.d == 128)
        k_quant_vt<128><<<g2, 256, 0, s>>>((const __nv_bfloat16*)v, p.d_perm, sigma, (int)p.N, p.H, (int)p.nb,
                                           (uint8_t*)vt);
    else
        k_quant_vt<64><<<g2, 256, 0, s>>>((const __nv_bfloat16*)v, p.d_perm, sigma, (int)p.N, p.H, (int)p.nb,
                                          (uint8_t*)vt);
    return cudaGetLastError();
}

}  // namespace bsa
