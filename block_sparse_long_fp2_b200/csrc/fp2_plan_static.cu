// fp2_plan_static: fp2_plan for callers that cannot allocate device memory.
//
// fp2_plan needs a caller-provided scratch workspace.  Some callers have no
// way to provide one: a serving process that has already handed (nearly)
// all device memory to its own KV-cache pool or caching allocator, so a
// further cudaMalloc would fail or fragment that pool; or a host program
// that only receives device pointers from another runtime and owns no
// device allocator at all.  This entry point runs the same planning
// kernels with their scratch placed in a fixed-size array that lives in
// the library's device image (kStaticWorkspaceBytes below).  The array is
// created when the library is loaded onto a device and is held by every
// device that loads the library until the process exits.
#include "fp2_internal.h"

namespace fp2 {

namespace {

constexpr size_t kStaticWorkspaceBytes = FP2_STATIC_WORKSPACE_BYTES;

// The scratch array.  In host code this name is only a host-side stand-in
// for the symbol, not a device address: the device address is obtained with
// cudaGetSymbolAddress below and only that address is handed to kernels.
static __device__ __align__(256) unsigned char g_static_workspace[kStaticWorkspaceBytes];

// Device address of the array in the current device's context, or nullptr.
// It is looked up on every call rather than cached: after cudaDeviceReset or
// a re-created primary context the array lives at a new address, and a cached
// one would point into freed memory.  The lookup is a host-side table read.
void* static_workspace_address() {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_workspace) != cudaSuccess) return nullptr;
    return p;
}

}  // namespace

}  // namespace fp2

using namespace fp2;

extern "C" int fp2_plan_static(const fp2_problem* problem, const void* q, const void* k,
                               const void* v, void* plan, size_t plan_bytes, void* stream) {
    Layout L;
    int rc = compute_layout(problem, &L);
    if (rc != FP2_OK) return rc;
    if (!q || !k || !v || !plan) return FP2_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(k) |
         reinterpret_cast<uintptr_t>(v)) % 16 != 0 ||
        reinterpret_cast<uintptr_t>(plan) % 256 != 0)
        return FP2_ERR_INVALID_ARG;
    if (plan_bytes < L.pub.plan_bytes) return FP2_ERR_CAPACITY;
    if (L.pub.workspace_bytes > kStaticWorkspaceBytes) return FP2_ERR_CAPACITY;
    void* ws = static_workspace_address();
    if (!ws) return FP2_ERR_CUDA;
    // No part of the workspace has to start at zero: every kernel writes the
    // scratch entries it reads later in the same call.
    const Dims& D = L.dims;
    const char* qb = static_cast<const char*>(q) + (int64_t)D.G * D.head0 * D.d * 2;
    const char* kb = static_cast<const char*>(k) + (int64_t)D.head0 * D.d * 2;
    const char* vb = static_cast<const char*>(v) + (int64_t)D.head0 * D.d * 2;
    return launch_plan(L, problem, qb, kb, vb, plan_ptrs(L, plan), ws_ptrs(L, ws),
                       static_cast<cudaStream_t>(stream));
}
