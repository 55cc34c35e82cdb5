// moe_layer_forward_static: the layer for callers that cannot allocate device memory.
// The intermediates live in a scratch buffer owned by the library (a file-scope device
// array, present on every GPU that loads the library until the process exits), so the call
// allocates and frees nothing. See include/moe_b200.h for the limits and the sharing rules.
#include <mutex>

#include "common.cuh"

namespace {

static __device__ __align__(256) uint8_t g_static_scratch[MOE_STATIC_SCRATCH_BYTES];

// Device address of the scratch on each device, looked up once per device with that
// device current (the array's name in host code is only a stand-in for the symbol).
constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

moe_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) return MOE_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return MOE_OK;
}

}  // namespace

extern "C" moe_status moe_layer_forward_static(const moe_layer* L, const void* x, void* out,
                                               moe_stream_t stream) {
  moe_status s = moe_validate(L);
  if (s != MOE_OK) return s;
  const size_t need = moe_workspace_size(L);
  if (need == 0) return MOE_ERR_INVALID_ARG;
  if (need > MOE_STATIC_SCRATCH_BYTES) return MOE_ERR_TOO_LARGE;
  void* ws = nullptr;
  if ((s = scratch_address(&ws)) != MOE_OK) return s;
  // the synchronisation block from the routing tickets on (tickets, barrier word,
  // failure-injection words, h counters, tile counters) begins at zero; the status word is
  // kept until moe_static_device_status reads it (the array starts zeroed at load)
  uint8_t* sync = static_cast<uint8_t*>(ws) + moe::kSyncTicket;
  if (cudaMemsetAsync(sync, 0, moe::sync_bytes(L->d) - moe::kSyncTicket,
                      reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return MOE_ERR_CUDA;
  return moe_layer_forward(L, x, out, nullptr, nullptr, nullptr, nullptr, ws,
                           MOE_STATIC_SCRATCH_BYTES, stream);
}

extern "C" moe_status moe_static_device_status(int32_t* code, moe_stream_t stream) {
  if (!code) return MOE_ERR_INVALID_ARG;
  void* ws = nullptr;
  moe_status s = scratch_address(&ws);
  if (s != MOE_OK) return s;
  int32_t* dev = static_cast<int32_t*>(ws) + moe::kSyncStatus / sizeof(int32_t);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int32_t h = 0;
  if (cudaMemcpyAsync(&h, dev, sizeof(int32_t), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess ||
      cudaMemsetAsync(dev, 0, sizeof(int32_t), st) != cudaSuccess)
    return MOE_ERR_CUDA;
  *code = (h == moe::DEV_OK) ? MOE_OK : (h == moe::DEV_TIMEOUT ? MOE_ERR_TIMEOUT : MOE_ERR_DEVICE);
  return MOE_OK;
}
