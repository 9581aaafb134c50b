// static_ws.cu - moe_ffn_forward_static: the MoE FFN forward with its scratch in
// a fixed device array compiled into the library, for callers that cannot
// allocate device memory.
//
// Who needs it: code that runs where a device allocation is not allowed or not
// safe, for example an inference engine's enqueue hook or plugin that must not
// allocate, a serving runtime that reserves all device memory up front, or a
// caller that cannot afford the implicit device synchronisation an allocation
// may cause.  Those callers still pass the inputs and the output; only the
// workspace comes from here.
#include <string.h>

#include <mutex>

#include "common.cuh"

namespace {

// The scratch of every moe_ffn_forward_static call, on every device that loads
// the library, held until the process exits.  In host code this name is only a
// stand-in for the symbol; kernels receive the device address obtained below.
static __device__ __align__(256) unsigned char g_static_ws[MOEQ_STATIC_WS_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_dev_ptr[kMaxDevices] = {};
// The layer shape of the last call on each device: the fused decode kernels keep
// epoch-tagged words and counters in the workspace that are laid out by shape, so
// the array is cleared whenever the shape changes.
struct ShapeKey {
    int32_t H, E, K, I, Is, r, valid;
};
ShapeKey g_last[kMaxDevices] = {};

// Device address of g_static_ws on the current device, looked up once per device.
moe_status static_ws_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_dev_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_ws) != cudaSuccess || !p) {
            (void)cudaGetLastError();
            return MOE_ERR_CUDA;
        }
        g_dev_ptr[dev] = p;
    }
    *out = g_dev_ptr[dev];
    return MOE_OK;
}

}  // namespace

extern "C" moe_status moe_ffn_forward_static(const moe_layer* layer, const uint16_t* x, const int32_t* adapter_id,
                                             int32_t T, uint16_t* y, moe_stream stream) {
    // The same checks as moe_ffn_forward, with the same results, before anything is
    // enqueued: a rejected call leaves the array (and the status it holds) untouched.
    moe_status st = moeq::ffn_precheck(layer, x, y, T);
    if (st != MOE_OK) return st;
    const size_t need = moe_ffn_workspace_bytes(layer, T);
    if (need > (size_t)MOEQ_STATIC_WS_BYTES) return MOE_ERR_WORKSPACE;
    if (T == 0) return MOE_OK;
    void* ws = nullptr;
    st = static_ws_address(&ws);
    if (st != MOE_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
    const ShapeKey key = {layer->hidden, layer->n_experts, layer->top_k, layer->inter,
                          layer->s_gate.packed ? layer->shared_inter : 0, layer->n_adapters > 0 ? layer->rank : 0, 1};
    bool same;
    {
        std::lock_guard<std::mutex> lock(g_mu);
        same = memcmp(&g_last[dev], &key, sizeof(key)) == 0;
        g_last[dev] = key;
    }
    // The array keeps the previous call's contents.  A call with the shape of the
    // previous one needs only the status word cleared (the decode counters and tagged
    // words carry over by design); a new shape starts from a cleared array.
    if (cudaMemsetAsync(ws, 0, same ? sizeof(int32_t) : (size_t)MOEQ_STATIC_WS_BYTES, s) != cudaSuccess)
        return MOE_ERR_CUDA;
    return moe_ffn_forward(layer, x, adapter_id, T, y, ws, need, stream);
}

extern "C" moe_status moe_ffn_static_device_status(moe_stream stream, int32_t* status) {
    if (!status) return MOE_ERR_INVALID_ARG;
    void* ws = nullptr;
    moe_status st = static_ws_address(&ws);
    if (st != MOE_OK) return st;
    return moe_get_device_status(ws, stream, status);
}
