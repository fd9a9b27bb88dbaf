// fg_ragged_attention_noalloc: the attention pass without any allocation.
//
// Some callers cannot allocate device memory at the point where they run the
// pass: a serving loop whose memory is fully reserved up front (the KV pool
// takes all of HBM but a fixed margin), code running under an allocator or
// policy that forbids cudaMalloc/cudaFree during a step, or an embedding that
// owns all device memory itself. fg_ragged_attention grows a per-batch split
// workspace and plan buffer with cudaMallocAsync when a pass needs more; this
// entry point instead uses two fixed arrays that live in the library's own
// device image (declared below), so it allocates nothing.
//
// The arrays are file-scope __device__ variables: every GPU that loads the
// library holds them (36 MiB) until the process exits. In host code their
// names are host-side stand-ins, not device addresses, so their device
// addresses are looked up once per device with cudaGetSymbolAddress (with
// that device current) and those addresses are what the kernels receive.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/fg.h"

namespace {

constexpr size_t kScratchFloats = size_t(8) << 20;  // split-KV partials: 8 Mi floats (32 MiB)
constexpr size_t kPlanBytes = size_t(4) << 20;      // work plan: 4 MiB

static __device__ __align__(256) float g_scratch_ws[kScratchFloats];
static __device__ __align__(256) unsigned char g_scratch_plan[kPlanBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
float* g_ws_addr[kMaxDevices] = {};
void* g_plan_addr[kMaxDevices] = {};

}  // namespace

fg_status fg_attention_launch_fixed(const fg_kv_cache* c, fg_ragged_batch* b, const void* q_rot,
                                    void* out, int32_t n_q_heads, float softmax_scale,
                                    int32_t window, cudaStream_t strm, float* ws,
                                    size_t ws_floats, void* plan_dev, size_t plan_bytes);
fg_status fg_set_error(fg_status st, const char* msg);

extern "C" fg_status fg_ragged_attention_noalloc(const fg_kv_cache* cache, fg_ragged_batch* batch,
                                                 const void* q_rot, void* out, int32_t n_q_heads,
                                                 float softmax_scale, int32_t sliding_window,
                                                 void* stream) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return fg_set_error(FG_ERR_CUDA, "fg_ragged_attention_noalloc: no usable current device");
  float* ws = nullptr;
  void* plan = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_ws_addr[dev]) {
      // first call on this device: resolve the arrays' device addresses
      void* w = nullptr;
      void* p = nullptr;
      cudaError_t e = cudaGetSymbolAddress(&w, g_scratch_ws);
      if (e == cudaSuccess) e = cudaGetSymbolAddress(&p, g_scratch_plan);
      if (e != cudaSuccess)
        return fg_set_error(FG_ERR_CUDA, "fg_ragged_attention_noalloc: cudaGetSymbolAddress failed");
      g_ws_addr[dev] = static_cast<float*>(w);
      g_plan_addr[dev] = p;
    }
    ws = g_ws_addr[dev];
    plan = g_plan_addr[dev];
  }
  return fg_attention_launch_fixed(cache, batch, q_rot, out, n_q_heads, softmax_scale,
                                   sliding_window, static_cast<cudaStream_t>(stream), ws,
                                   kScratchFloats, plan, kPlanBytes);
}
