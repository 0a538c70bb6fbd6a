// loki_decode_attention_noalloc: the decode step with its scratch memory taken
// from a fixed-size array compiled into this library instead of a
// caller-provided workspace.
//
// Who needs it: callers that cannot allocate device memory themselves --
// plugins hosted by a framework that owns every device allocation and offers
// no allocator to them, and latency-critical threads that must not call
// cudaMalloc / cudaFree because those calls can synchronise the whole device.
// Such callers still pass their inputs and outputs; only the scratch (rotated
// queries, scores and attention partials) comes from here.
//
// Costs and limits:
//   * the array (kScratchBytes, 32 MiB) is device memory that every GPU which
//     loads this library holds until the process exits;
//   * a call whose decode needs more scratch than that is rejected with
//     LOKI_ERR_UNSUPPORTED before anything is launched;
//   * every call shares the one array: calls that overlap on the GPU (on
//     different streams, or from different threads without ordering) race
//     on it. The decode path writes all scratch it reads, so nothing has to
//     start at zero, and leftovers of a previous call do not matter;
//   * the first call on each device looks up the array's device address
//     (cudaGetSymbolAddress, with that device current) and caches it; make
//     that first call before any stream capture begins.
#include <mutex>

#include "../../include/loki.h"
#include "launch.h"

namespace {

constexpr size_t kScratchBytes = size_t(32) << 20;
constexpr int kMaxDevices = 64;

// In host code this name is only a host-side handle to the array, not a
// device address: the device address comes from cudaGetSymbolAddress.
__device__ __align__(256) unsigned char g_scratch[kScratchBytes];

std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

}  // namespace

extern "C" loki_status loki_decode_attention_noalloc(const void* q, const void* Kt_cache,
                                                     const void* V_cache, const float* P, int B,
                                                     int H_q, int H_kv, int64_t S, int64_t S_max,
                                                     int D, int d, int64_t k, float scale,
                                                     loki_dtype dt, void* out,
                                                     int32_t* selected_idx, void* stream) {
    const size_t need = loki_decode_workspace_size(B, H_q, H_kv, S, D, d, k);
    if (need > kScratchBytes) {
        loki::set_last_error("loki_decode_attention_noalloc: this decode needs more scratch than "
                             "the built-in 32 MiB array holds; use loki_decode_attention with a "
                             "caller-provided workspace");
        return LOKI_ERR_UNSUPPORTED;
    }
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        loki::set_last_error("loki_decode_attention_noalloc: no usable current CUDA device");
        return LOKI_ERR_CUDA;
    }
    void* scratch = nullptr;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        if (g_scratch_ptr[dev] == nullptr) {
            e = cudaGetSymbolAddress(&g_scratch_ptr[dev], g_scratch);
            if (e != cudaSuccess) {
                g_scratch_ptr[dev] = nullptr;
                loki::set_last_error("loki_decode_attention_noalloc: cudaGetSymbolAddress of the "
                                     "built-in scratch array failed");
                return LOKI_ERR_CUDA;
            }
        }
        scratch = g_scratch_ptr[dev];
    }
    return loki_decode_attention(q, Kt_cache, V_cache, P, B, H_q, H_kv, S, S_max, D, d, k, scale,
                                 dt, out, selected_idx, scratch, kScratchBytes, stream);
}
