// Fixed block masks produced on the device, as CSR for bsa_sparse_attn.
//
// Window plus rotating global anchors (LVSA wiki page, "TL;DR" and "Key
// points": a structured local window pattern plus global anchor blocks that
// shift across diffusion timesteps).  On the frame-major token order a block
// covers a contiguous range of latent frames, so the window part of a row is
// one contiguous range of key blocks [jlo, jhi]; the anchors
// {(step + m*floor(nb/n_anchor)) mod nb} are merged in ascending order.
//   k_mask_count  per row: window range + anchors outside it -> count
//   (scan)        row_ptr, nnz (the routing CSR scan)
//   k_mask_fill   per row: ascending unique columns
#include "bsa_internal.cuh"

namespace bsa {
namespace {

constexpr int kMaxAnchors = kMaxMaskAnchors;

struct WindowRow {
    int jlo, jhi;
};

// Key blocks whose frame range comes within `radius` frames of block i's.
__device__ __forceinline__ WindowRow window_range(int i, int N, int block, int hw, int nb, int radius) {
    const int first_i = (i * block) / hw;
    const int last_i = (min(N, (i + 1) * block) - 1) / hw;
    const long long F = (long long)first_i - radius;     // need last_j >= F
    const long long Lf = (long long)last_i + radius;      // need first_j <= Lf
    int jlo = 0;
    if (F > 0) {
        // last_j >= F  <=>  min(N, (j+1)*block) - 1 >= F*hw  <=>  (j+1)*block >= F*hw + 1
        jlo = (int)((F * hw + 1 + block - 1) / block) - 1;
        jlo = max(0, min(jlo, nb - 1));
    }
    // first_j <= Lf  <=>  j*block < (Lf+1)*hw
    long long jh = ((Lf + 1) * hw + block - 1) / block - 1;
    const int jhi = (int)(jh < nb - 1 ? jh : nb - 1);
    return {jlo, jhi};
}

// Sorted unique anchors of one step; returns their number.
__device__ __forceinline__ int anchors(int nb, int n_anchor, int step, int* a) {
    const int stride = nb / n_anchor;
    int n = 0;
    for (int m = 0; m < n_anchor; ++m) {
        const int v = (int)(((long long)step + (long long)m * stride) % nb);
        int pos = n;
        bool dup = false;
        for (int t = 0; t < n; ++t) {
            if (a[t] == v) { dup = true; break; }
        }
        if (dup) continue;
        while (pos > 0 && a[pos - 1] > v) { a[pos] = a[pos - 1]; --pos; }
        a[pos] = v;
        ++n;
    }
    return n;
}

__global__ void k_mask_count(int64_t rows, int N, int block, int hw, int nb, int radius, int n_anchor, int step,
                             int32_t* __restrict__ counts) {
    const int64_t r = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (r >= rows) return;
    const int i = (int)(r % nb);
    const WindowRow w = window_range(i, N, block, hw, nb, radius);
    int a[kMaxAnchors];
    const int na = n_anchor > 0 ? anchors(nb, n_anchor, step, a) : 0;
    int c = w.jhi - w.jlo + 1;
    for (int t = 0; t < na; ++t) c += (a[t] < w.jlo || a[t] > w.jhi);
    counts[r] = c;
}

__global__ void k_mask_fill(int64_t rows, int N, int block, int hw, int nb, int radius, int n_anchor, int step,
                            const int32_t* __restrict__ row_ptr, int32_t* __restrict__ col_idx, int64_t col_cap) {
    const int64_t r = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (r >= rows) return;
    const int i = (int)(r % nb);
    const WindowRow w = window_range(i, N, block, hw, nb, radius);
    int a[kMaxAnchors];
    const int na = n_anchor > 0 ? anchors(nb, n_anchor, step, a) : 0;
    int64_t pos = row_ptr[r];
    int t = 0;
    auto put = [&](int j) { if (pos < col_cap) col_idx[pos] = j; ++pos; };
    for (; t < na && a[t] < w.jlo; ++t) put(a[t]);
    for (int j = w.jlo; j <= w.jhi; ++j) put(j);
    for (; t < na; ++t)
        if (a[t] > w.jhi) put(a[t]);
}

}  // namespace

cudaError_t launch_mask_window_anchor(const bsa_plan& p, int radius, int n_anchor, int step, int32_t* counts,
                                      int32_t* row_ptr, int32_t* col_idx, int64_t col_cap, int64_t* nnz,
                                      cudaStream_t s) {
    const int hw = p.Hs * p.Ws;
    const int t = 256;
    const unsigned g = (unsigned)((p.rows + t - 1) / t);
    k_mask_count<<<g, t, 0, s>>>(p.rows, (int)p.N, p.block, hw, (int)p.nb, radius, n_anchor, step, counts);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    e = launch_scan_counts(p, counts, row_ptr, nullptr, nnz, col_cap, s);
    if (e != cudaSuccess) return e;
    k_mask_fill<<<g, t, 0, s>>>(p.rows, (int)p.N, p.block, hw, (int)p.nb, radius, n_anchor, step, row_ptr, col_idx,
                                col_cap);
    return cudaGetLastError();
}

}  // namespace bsa
