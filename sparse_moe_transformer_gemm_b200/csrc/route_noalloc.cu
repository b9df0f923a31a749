// route_noalloc.cu -- moe_route_noalloc: the router for callers that cannot
// allocate device memory.
//
// moe_route needs device scratch besides its inputs and outputs: the fp32
// logits of every token ([T, E]) and one arrival counter per group of 8
// tokens. It normally lives in the caller's workspace. Some callers cannot
// provide one: code that runs where an allocation is not allowed or not
// available (a host framework that hands out no device memory to plugins, a
// latency-critical loop where cudaMalloc may synchronise the device), or a
// caller that simply has nowhere to keep a workspace between calls. For them
// this entry point keeps the scratch in a fixed device array compiled into the
// library (MOE_NOALLOC_SCRATCH_BYTES, 2 MiB), which every GPU that loads the
// library holds until the process exits.
//
// Set-up: the first call on each device, with that device current, looks up
// the array's device address (cudaGetSymbolAddress) and remembers it; make
// that first call before any stream capture. Host code cannot pass the array's
// name to a kernel directly -- on the host it denotes a host-side stand-in,
// not the device memory.
//
// Sharing: every call uses the same array, which keeps the last call's
// contents. The counters are cleared at the start of every call; the logits
// are fully rewritten. Calls whose work overlaps on the GPU (different
// streams, or several host threads) race on the array and must be serialised
// by the caller.
#include <mutex>

#include "internal.h"

namespace {

constexpr size_t kScratchBytes = MOE_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_route_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_scratch_addr[kMaxDevices];

// Device address of g_route_scratch on the current device, looked up once.
int scratch_address(void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (g_scratch_addr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_route_scratch) != cudaSuccess || p == nullptr)
            return MOE_ERR_CUDA;
        g_scratch_addr[dev] = p;
    }
    *out = g_scratch_addr[dev];
    return MOE_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" int moe_route_noalloc(const moe_config* cfg, const void* x, const void* w_gate,
                                 const float* gate_bias, int32_t* topk_idx, float* topk_w,
                                 void* stream) {
    if (!cfg) return MOE_ERR_INVALID_ARG;
    if (moe_workspace_size(cfg) == 0) return MOE_ERR_UNSUPPORTED_SHAPE;  // shape and flag checks
    if (!x || !w_gate || !topk_idx || !topk_w || !aligned16(x) || !aligned16(w_gate))
        return MOE_ERR_INVALID_ARG;
    const size_t counter_bytes = moe::align256(sizeof(int32_t) * moe::n_router_groups(*cfg));
    const size_t logit_bytes = sizeof(float) * (size_t)cfg->T * cfg->E;
    if (counter_bytes + logit_bytes > kScratchBytes) return MOE_ERR_UNSUPPORTED_SHAPE;
    void* base = nullptr;
    const int rc = scratch_address(&base);
    if (rc != MOE_OK) return rc;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int32_t* counters = static_cast<int32_t*>(base);
    float* logits = reinterpret_cast<float*>(static_cast<char*>(base) + counter_bytes);
    if (cudaMemsetAsync(counters, 0, counter_bytes, s) != cudaSuccess) return MOE_ERR_CUDA;
    return moe::launch_router(*cfg, x, w_gate, gate_bias, nullptr, nullptr, 0.f, 0, topk_idx,
                              topk_w, logits, nullptr, counters, 1, s) ==
                   cudaSuccess
               ? MOE_OK
               : MOE_ERR_CUDA;
}
