// Slack-aware sparse augmentation, the in-place mechanism (FVAttn review,
// section 3 "Stage 3: Slack-Aware Sparse Augmentation" and the SASA algorithm
// flow of section 5: unselected high-value blocks are added from the already
// sorted key-block importance order, with no re-sorting and no QK scoring).
//   k_aug_count  n_out = min(nb, n_in + extra[head])  per row
//   (scan)       row_ptr_out, nnz_out, L_h_out (Eq. 1)
//   k_aug_fill   col_idx_out row = the first n_out blocks of the row's order
#include "bsa_internal.cuh"

namespace bsa {
namespace {

__global__ void k_aug_count(const int32_t* __restrict__ row_ptr, const int32_t* __restrict__ extra, int64_t rows,
                            int nb, int32_t* __restrict__ counts, int32_t* err) {
    const int64_t r = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (r >= rows) return;
    int n = row_ptr[r + 1] - row_ptr[r];
    if (n < 0 || n > nb) {
        record_error(err, BSA_EDEVICE, (int)r);
        n = n < 0 ? 0 : nb;
    }
    const int a = extra[r / nb];
    counts[r] = min(nb, n + (a > 0 ? a : 0));
}

__global__ void k_aug_fill(const uint16_t* __restrict__ order, const int32_t* __restrict__ counts,
                           const int32_t* __restrict__ row_ptr_out, int32_t* __restrict__ col_idx, int64_t rows,
                           int nb, int64_t col_cap) {
    const int64_t r = (int64_t)blockIdx.x * (blockDim.x / 32) + threadIdx.x / 32;
    if (r >= rows) return;
    const int n = counts[r];
    const int64_t base = row_ptr_out[r];
    const uint16_t* src = order + r * nb;
    for (int t = threadIdx.x % 32; t < n; t += 32)
        if (base + t < col_cap) col_idx[base + t] = src[t];
}

}  // namespace

cudaError_t launch_augment(const bsa_plan& p, const int32_t* row_ptr, const uint16_t* order, const int32_t* extra,
                           int32_t* counts, int32_t* row_ptr_out, int32_t* col_idx_out, int64_t col_cap,
                           float* L_h_out, int64_t* nnz_out, cudaStream_t s) {
    const int t = 256;
    k_aug_count<<<(unsigned)((p.rows + t - 1) / t), t, 0, s>>>(row_ptr, extra, p.rows, (int)p.nb, counts, p.d_err);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    e = launch_scan_counts(p, counts, row_ptr_out, L_h_out, nnz_out, col_cap, s);
    if (e != cudaSuccess) return e;
    if (col_cap == 0) return cudaSuccess;
    const int rows_per_cta = 8;
    k_aug_fill<<<(unsigned)((p.rows + rows_per_cta - 1) / rows_per_cta), 32 * rows_per_cta, 0, s>>>(
        order, counts, row_ptr_out, col_idx_out, p.rows, (int)p.nb, col_cap);
    return cudaGetLastError();
}

}  // namespace bsa
