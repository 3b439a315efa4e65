// sdk_decode_attn_static: the decode-attention call of sdk_decode_attn with
// its workspace in a fixed array of the library's own device memory, so that
// the call allocates nothing and takes no workspace argument.
//
// Who needs it: callers that cannot allocate device memory at the point
// where they decode.  A serving loop whose device memory is budgeted and
// handed out before the first request has no allocator on its decode
// thread; a plain C host embedding the library may hold no device
// allocator at all.  A cudaMalloc/cudaFree there would also synchronise the
// device and stall every other stream of the step.  Such a caller gets a
// workspace of fixed size, SDK_DECODE_STATIC_WS_BYTES per device, set aside
// when the library's device code is loaded.
//
// The arithmetic is exactly that of sdk_decode_attn: this file only finds
// the array's address and forwards the call.
#include <mutex>

#include "sdk_internal.cuh"

// One workspace per device (a __device__ array exists once in every
// context that loads this module).  Its layout is the decode workspace of
// sdk_decode_layout_of.  What must start at zero: the first two words of
// the 256-byte header (recorded device-side failure and its detail); a
// __device__ array is zero when the module loads, and every call that
// passes status_out copies those words out and zeroes them again.  The
// decode kernels write every other region before reading it.
static __device__ __align__(256) unsigned char g_decode_static_ws[SDK_DECODE_STATIC_WS_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_mu;
// Per device: the id of the context the address was looked up in, and the
// address.  A __device__ array lives in the module loaded into one
// context; after cudaDeviceReset (or anything else that destroys the
// primary context) the module is loaded again, possibly at another
// address, so the address is looked up again whenever the current
// context's id differs (context ids are unique within a process; a
// context handle may be reused).
unsigned long long g_ws_ctx[kMaxDevices] = {};
void* g_ws_ptr[kMaxDevices] = {};

// cuCtxGetCurrent and cuCtxGetId through the runtime's driver entry points
// (null when the driver does not offer them).
using CtxGetCurrentFn = int (*)(void**);
using CtxGetIdFn = int (*)(void*, unsigned long long*);
template <class Fn>
Fn driver_fn(const char* name) {
  void* ptr = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPointByVersion(name, &ptr, 12000, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess)
    return nullptr;
  return reinterpret_cast<Fn>(ptr);
}

// Id of the calling thread's current context (0 if none or unknown).
unsigned long long current_ctx_id() {
  static CtxGetCurrentFn get_ctx = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
  static CtxGetIdFn get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
  void* ctx = nullptr;
  unsigned long long id = 0ull;
  if (get_ctx == nullptr || get_id == nullptr || get_ctx(&ctx) != 0 || ctx == nullptr) return 0ull;
  if (get_id(ctx, &id) != 0) return 0ull;
  return id;
}

// Address of the array in the current device's current context, looked up
// on the first call in that context (the lookup loads the module if it is
// not loaded yet, and makes the device's primary context current).
sdk_status static_workspace(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SDK_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return SDK_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  unsigned long long id = current_ctx_id();
  if (id == 0ull || g_ws_ptr[dev] == nullptr || g_ws_ctx[dev] != id) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress((void**)&ptr, g_decode_static_ws) != cudaSuccess || ptr == nullptr)
      return SDK_ERR_CUDA;
    if (id == 0ull) id = current_ctx_id();
    if (id == 0ull) return SDK_ERR_CUDA;
    g_ws_ptr[dev] = ptr;
    g_ws_ctx[dev] = id;
  }
  *out = g_ws_ptr[dev];
  return SDK_OK;
}

}  // namespace

extern "C" {

sdk_status sdk_decode_attn_static(const float* q, int32_t B, int32_t Hq, int32_t Hkv,
                                  int32_t head_dim, const void* dict_k, const void* dict_v,
                                  int32_t n_atoms, const uint32_t* k_lo, const uint32_t* k_full,
                                  const uint32_t* v_full, int64_t cap, const int32_t* lens_host,
                                  int32_t klow, int32_t khigh, int32_t top_num, int32_t top_den,
                                  int32_t flags, float scale, float* out,
                                  uint32_t* status_out, sdk_stream_t stream) {
  // the lengths decide the workspace size, so they are checked first
  if (lens_host == nullptr || B < 1 || B > SDK_MAX_BATCH || cap < 1) return SDK_ERR_INVALID_ARG;
  int64_t max_len = 1;
  for (int b = 0; b < B; ++b) {
    if (lens_host[b] < 1 || lens_host[b] > cap) return SDK_ERR_INVALID_ARG;
    if (lens_host[b] > max_len) max_len = lens_host[b];
  }
  // need == 0 means an invalid shape, which sdk_decode_attn reports below
  const size_t need = sdk_decode_workspace_bytes(B, Hq, head_dim, n_atoms, max_len);
  if (need > (size_t)SDK_DECODE_STATIC_WS_BYTES) return SDK_ERR_CAPACITY;
  if (status_out != nullptr && (reinterpret_cast<uintptr_t>(status_out) & 3u) != 0u)
    return SDK_ERR_INVALID_ARG;
  void* ws = nullptr;
  sdk_status s = static_workspace(&ws);
  if (s != SDK_OK) return s;
  s = sdk_decode_attn(q, B, Hq, Hkv, head_dim, dict_k, dict_v, n_atoms, k_lo, k_full, v_full, cap,
                      lens_host, klow, khigh, top_num, top_den, flags, scale, out, ws,
                      (size_t)SDK_DECODE_STATIC_WS_BYTES, stream);
  if (s != SDK_OK || status_out == nullptr) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(status_out, ws, 2 * sizeof(uint32_t), cudaMemcpyDeviceToDevice, st) !=
          cudaSuccess ||
      cudaMemsetAsync(ws, 0, 2 * sizeof(uint32_t), st) != cudaSuccess)
    return SDK_ERR_CUDA;
  return SDK_OK;
}

}  // extern "C"
