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
// that first call before any stream capture. Later calls on a stream that is
// not being captured look the address up again (cheap once the module is
// loaded), so a device reset and a new context do not leave a stale address;
// a call under capture uses the remembered one. Host code cannot pass the
// array's name to a kernel directly -- on the host it denotes a host-side
// stand-in, not the device memory.
//
// Kernel: the CUDA-core router with the K split that moe_route gives it, so
// wherever moe_route runs that router (T <= 128, or shapes the tensor-core
// router does not take) the two calls give bitwise the same indices and
// weights. For T >= 129 on shapes the tensor-core router takes, moe_route
// runs that one instead; its fp32 logits sum in another order, so the choice
// agrees on every token whose k-th/(k+1)-th score gap is at least ~1e-5 and
// the weights to ~2e-5 relative. The tensor-core router is not used here: it
// reports a bounded wait that gave up through a status word, and this entry
// point has no workspace to carry one back to the caller.
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

// Device address of g_route_scratch on the current device: looked up on every
// call outside stream capture, remembered for calls under capture.
int scratch_address(cudaStream_t s, void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_ERR_CUDA;
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(s, &cap) != cudaSuccess) return MOE_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_setup_mutex);
    if (cap == cudaStreamCaptureStatusNone || g_scratch_addr[dev] == nullptr) {
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
    // moe_route's K split of the CUDA-core router: the same partial sums in the
    // same order (at most 16 slices; for T > 128 at E = 192 it is 1)
    const int ksplit = moe::router_ksplit(*cfg);
    const size_t counter_bytes = moe::align256(sizeof(int32_t) * moe::n_router_groups(*cfg));
    const size_t logit_bytes = sizeof(float) * (size_t)ksplit * cfg->T * cfg->E;
    if (counter_bytes + logit_bytes > kScratchBytes) return MOE_ERR_UNSUPPORTED_SHAPE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    void* base = nullptr;
    const int rc = scratch_address(s, &base);
    if (rc != MOE_OK) return rc;
    int32_t* counters = static_cast<int32_t*>(base);
    float* logits = reinterpret_cast<float*>(static_cast<char*>(base) + counter_bytes);
    if (cudaMemsetAsync(counters, 0, counter_bytes, s) != cudaSuccess) return MOE_ERR_CUDA;
    return moe::launch_router(*cfg, x, w_gate, gate_bias, nullptr, nullptr, 0.f, 0, topk_idx,
                              topk_w, logits, nullptr, counters, ksplit, s) == cudaSuccess
               ? MOE_OK
               : MOE_ERR_CUDA;
}
