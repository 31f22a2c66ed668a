// bsa_route_static: the routing entry point for callers that cannot allocate
// device memory when they route -- for example a host that has handed all
// device memory to its own fixed arena or caching allocator.
//
// It runs exactly the kernels of bsa_route, but their scratch (pooled Q/K,
// block scores, sorted indices, counts) lives in one file-scope device array
// of kRouteScratchBytes that every GPU loading this library holds until the
// process exits.  The caller still owns q, k and all outputs.
#include <mutex>

#include "bsa_internal.cuh"

namespace bsa {
namespace {

constexpr size_t kRouteScratchBytes = 32ull << 20;     // 32 MiB
constexpr int kMaxDevices = 64;

// Host code must not take this array's address directly: on the host the name
// is only a stand-in.  The device address is fetched once per device below.
static __device__ __align__(256) unsigned char g_route_scratch[kRouteScratchBytes];

// Cached per device for the life of the process.  The address belongs to the
// device's primary context: a cudaDeviceReset (or anything else that destroys
// that context) leaves it stale, and the header tells callers not to route
// through this entry point after such a reset.
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_route_scratch on the current device (set up on first use).
int scratch_for_current_device(int dev, void** out) {
    if (dev < 0 || dev >= kMaxDevices) return BSA_EUNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_ptr[dev]) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_route_scratch) != cudaSuccess || !ptr) return BSA_ECUDA;
        g_scratch_ptr[dev] = ptr;
    }
    *out = g_scratch_ptr[dev];
    return BSA_OK;
}

}  // namespace
}  // namespace bsa

using namespace bsa;

extern "C" int bsa_route_static(const bsa_plan* p, const void* q, const void* k, int dtype, float pval, int k_floor,
                                int32_t* row_ptr, int32_t* col_idx, int64_t col_cap, float* L_h, int64_t* nnz,
                                void* stream) {
    if (!p || !q || !k || !row_ptr || !L_h || !nnz) return BSA_EINVAL;
    if (col_cap < 0 || (col_cap > 0 && !col_idx)) return BSA_EINVAL;
    if (dtype != BSA_BF16 && dtype != BSA_F32) return BSA_EINVAL;
    if (!(pval > 0.0f) || !(pval <= 1.0f) || k_floor < 0) return BSA_EINVAL;
    if (((uintptr_t)q | (uintptr_t)k) % 16 != 0 || (uintptr_t)row_ptr % 4 != 0 ||
        (col_idx && (uintptr_t)col_idx % 4 != 0) || (uintptr_t)L_h % 4 != 0 || (uintptr_t)nnz % 8 != 0)
        return BSA_EINVAL;
    if (p->nb > kMaxRouteBlocks) return BSA_EUNSUPPORTED;
    const RouteWs L = route_ws_layout(*p);
    if (L.total > kRouteScratchBytes) return BSA_EWORKSPACE;      // shape too large for the fixed scratch
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return BSA_ECUDA;
    if (dev != p->device) return BSA_EINVAL;
    void* scratch = nullptr;
    if (int rc = scratch_for_current_device(dev, &scratch)) return rc;
    // Every region below is fully written before it is read, so stale contents
    // left by an earlier call need no clearing.
    cudaStream_t s = (cudaStream_t)stream;
    char* base = (char*)scratch;
    double* qbar = (double*)(base + L.qbar);
    double* kbar = (double*)(base + L.kbar);
    double* scores = (double*)(base + L.scores);
    uint16_t* sorted = (uint16_t*)(base + L.sorted);
    int32_t* counts = (int32_t*)(base + L.counts);
    if (launch_route_stages(*p, q, k, dtype, (double)pval, k_floor, qbar, kbar, scores, sorted, counts, s) !=
        cudaSuccess)
        return BSA_ECUDA;
    if (launch_csr(*p, counts, sorted, row_ptr, col_idx, col_cap, L_h, nnz, s) != cudaSuccess) return BSA_ECUDA;
    return BSA_OK;
}
