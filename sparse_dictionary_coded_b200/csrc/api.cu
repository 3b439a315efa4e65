// C ABI of libsdk.so: argument checks, workspace carving and stream-ordered
// launches.  The operations are defined in include/sdk.h.
#include <atomic>
#include <cmath>
#include <cstring>

#include "sdk_internal.cuh"

namespace sdk {



namespace {
std::atomic<unsigned long long> g_exchange_wait_ns{1000000000ull};
}
unsigned long long exchange_wait_ns() { return g_exchange_wait_ns.load(std::memory_order_relaxed); }
unsigned long long set_exchange_wait_ns(unsigned long long ns) {
  return g_exchange_wait_ns.exchange(ns, std::memory_order_relaxed);
}

int num_sms() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (cache[dev] == 0) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0)
      v = 148;
    cache[dev] = v;
  }
  return cache[dev];
}

static unsigned long long device_bit() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0ull;
  return 1ull << dev;
}

bool device_needs_setup(const unsigned long long* flags) {
  const unsigned long long bit = device_bit();
  return bit == 0ull || (__atomic_load_n(flags, __ATOMIC_ACQUIRE) & bit) == 0ull;
}

void device_setup_done(unsigned long long* flags) {
  __atomic_fetch_or(flags, device_bit(), __ATOMIC_RELEASE);
}

}  // namespace sdk

using namespace sdk;

namespace {

bool aligned(const void* p, size_t a) {
  return (reinterpret_cast<uintptr_t>(p) % a) == 0;
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

sdk_status check_encode_args(const void* x, int32_t x_dtype, int64_t n_vec,
                             int32_t head_dim, const void* dict, int32_t n_atoms,
                             int32_t k_atoms, const uint32_t* codes_out,
                             const void* workspace) {
  if (n_vec < 0 || n_atoms < 1 || n_atoms > SDK_MAX_ATOMS || k_atoms < 1 ||
      k_atoms > SDK_K_ATOMS)
    return SDK_ERR_INVALID_ARG;
  if (x_dtype != SDK_F32 && x_dtype != SDK_BF16) return SDK_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return SDK_ERR_UNSUPPORTED;
  if (workspace == nullptr || !aligned(workspace, SDK_WS_ALIGN)) return SDK_ERR_INVALID_ARG;
  if (n_vec == 0) return SDK_OK;
  if (x == nullptr || dict == nullptr || codes_out == nullptr) return SDK_ERR_INVALID_ARG;
  if (!aligned(dict, 16) || !aligned(x, x_dtype == SDK_F32 ? 4 : 2) || !aligned(codes_out, 4))
    return SDK_ERR_INVALID_ARG;
  return SDK_OK;
}

}  // namespace

extern "C" {

const char* sdk_status_string(int status) {
  switch (status) {
    case SDK_OK: return "SDK_OK";
    case SDK_ERR_INVALID_ARG: return "SDK_ERR_INVALID_ARG: invalid argument";
    case SDK_ERR_UNSUPPORTED: return "SDK_ERR_UNSUPPORTED: configuration not built";
    case SDK_ERR_CAPACITY: return "SDK_ERR_CAPACITY: capacity or workspace too small";
    case SDK_ERR_CUDA: return "SDK_ERR_CUDA: CUDA runtime or launch failure";
    case SDK_ERR_TIMEOUT: return "SDK_ERR_TIMEOUT: bounded device wait expired";
    case SDK_ERR_DEVICE_CHECK: return "SDK_ERR_DEVICE_CHECK: device-side check failed";
    default: return "SDK_ERR_UNKNOWN";
  }
}

int32_t sdk_version(void) { return 2; }

uint64_t sdk_set_exchange_timeout_ns(uint64_t ns) { return sdk::set_exchange_wait_ns(ns); }

size_t sdk_encode_workspace_bytes(int64_t n_vec, int32_t head_dim, int32_t n_atoms) {
  if (n_vec < 0) n_vec = 0;
  size_t scratch = encode_tc_scratch_bytes(n_vec, head_dim, n_atoms);
  if (n_vec >= 1 && n_vec <= kSmallEncodeRows && encode_small_scratch_bytes() > scratch)
    scratch = encode_small_scratch_bytes();
  return align_up(sizeof(WsHeader), 256) + align_up(scratch, 256);
}

// Runs the encoder with an explicit header and scratch area (the scratch is
// what the tensor-core encoder needs beyond its inputs and outputs).
// Words between consecutive tokens' records: 32 when k_full and v_full point
// into one interleaved array (v_full = k_full + 16 words), else 16.
static int record_stride(const uint32_t* k_full, const uint32_t* v_full) {
  return v_full == k_full + SDK_K_ATOMS ? 2 * SDK_K_ATOMS : SDK_K_ATOMS;
}

static sdk_status encode_core(bool allow_tc, const EncodeParams& p, int head_dim, void* scratch,
                              size_t scratch_bytes, cudaStream_t st) {
  if (p.n_vec == 0) return SDK_OK;
  if (allow_tc && p.n_vec <= kSmallEncodeRows) {
    SmallEncode e;
    memset(&e, 0, sizeof(e));
    e.p[0] = p;
    e.streams = 1;
    e.head_dim = head_dim;
    bool taken = false;
    sdk_status s = launch_encode_small(e, scratch, scratch_bytes, st, &taken);
    if (taken) return s;
  }
  if (allow_tc) {
    bool taken = false;
    sdk_status s = launch_encode_tc(&p, 1, head_dim, scratch, scratch_bytes, st, &taken);
    if (taken) return s;
  }
  return launch_encode_simt(p, head_dim, st);
}

static sdk_status encode_impl(bool allow_tc, const void* x, int32_t x_dtype, int64_t n_vec,
                              int32_t head_dim, const void* dict, int32_t n_atoms,
                              int32_t k_atoms, uint32_t* codes_out, float* resid_sqnorm_out,
                              void* workspace, size_t ws_bytes, sdk_stream_t stream) {
  sdk_status s = check_encode_args(x, x_dtype, n_vec, head_dim, dict, n_atoms, k_atoms,
                                   codes_out, workspace);
  if (s != SDK_OK) return s;
  const size_t need = sdk_encode_workspace_bytes(n_vec, head_dim, n_atoms);
  if (ws_bytes < (allow_tc ? need : sizeof(WsHeader))) return SDK_ERR_CAPACITY;
  if (n_vec == 0) return SDK_OK;
  EncodeParams p;
  p.x = x;
  p.x_dtype = x_dtype;
  p.n_vec = n_vec;
  p.dict = reinterpret_cast<const uint16_t*>(dict);
  p.n = n_atoms;
  p.k_atoms = k_atoms;
  p.codes = codes_out;
  p.rsq = resid_sqnorm_out;
  p.hdr = reinterpret_cast<WsHeader*>(workspace);
  const size_t hb = align_up(sizeof(WsHeader), 256);
  return encode_core(allow_tc, p, head_dim, reinterpret_cast<char*>(workspace) + hb,
                     allow_tc ? need - hb : 0, reinterpret_cast<cudaStream_t>(stream));
}

sdk_status sdk_encode(const void* x, int32_t x_dtype, int64_t n_vec, int32_t head_dim,
                      const void* dict, int32_t n_atoms, int32_t k_atoms, uint32_t* codes_out,
                      float* resid_sqnorm_out, void* workspace, size_t ws_bytes,
                      sdk_stream_t stream) {
  return encode_impl(true, x, x_dtype, n_vec, head_dim, dict, n_atoms, k_atoms, codes_out,
                     resid_sqnorm_out, workspace, ws_bytes, stream);
}

sdk_status sdk_encode_simt(const void* x, int32_t x_dtype, int64_t n_vec, int32_t head_dim,
                           const void* dict, int32_t n_atoms, int32_t k_atoms,
                           uint32_t* codes_out, float* resid_sqnorm_out, void* workspace,
                           size_t ws_bytes, sdk_stream_t stream) {
  return encode_impl(false, x, x_dtype, n_vec, head_dim, dict, n_atoms, k_atoms, codes_out,
                     resid_sqnorm_out, workspace, ws_bytes, stream);
}

}  // extern "C"

// ------------------------------------------------------------------ append
namespace sdk {

struct ScatterParams {
  const uint32_t* codes;  // [nv][16]
  uint32_t* full;         // [B][Hkv][cap][16]
  uint32_t* lo;           // [B][Hkv][3][cap] or null
  int64_t cap;
  int Hkv, n_new, rs;
  int64_t nv;
  int lens[kMaxBatch];
};

__global__ void scatter_codes_kernel(ScatterParams p) {
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= p.nv * kAtoms) return;
  const int64_t v = e / kAtoms;
  const int j = (int)(e % kAtoms);
  const int64_t bk = v / p.n_new;
  const int i = (int)(v % p.n_new);
  const int b = (int)(bk / p.Hkv);
  const int64_t t = (int64_t)p.lens[b] + i;
  const uint32_t w = p.codes[e];
  p.full[(bk * p.cap + t) * p.rs + j] = w;
  if (p.lo != nullptr && j < kLoPlanes) p.lo[(bk * kLoPlanes + j) * p.cap + t] = w;
}

}  // namespace sdk

extern "C" {

// header, K and V code buffers [nv][16] each, then the encoder's scratch for
// both streams in one launch (or the small encoder's)
size_t sdk_append_workspace_bytes(int32_t B, int32_t Hkv, int32_t n_new, int32_t head_dim,
                                  int32_t n_atoms) {
  const int64_t nv = (int64_t)(B > 0 ? B : 0) * (Hkv > 0 ? Hkv : 0) * (n_new > 0 ? n_new : 0);
  size_t scratch = encode_tc_scratch_bytes(2 * nv, head_dim, n_atoms, 2);
  const size_t one = sdk_encode_workspace_bytes(nv, head_dim, n_atoms) - align_up(sizeof(WsHeader), 256);
  if (one > scratch) scratch = one;
  return align_up(sizeof(WsHeader), 256) + 2 * align_up((size_t)nv * kAtoms * 4, 256) +
         align_up(scratch, 256);
}

sdk_status sdk_append(const void* xk, const void* xv, int32_t x_dtype, int32_t B, int32_t Hkv,
                      int32_t n_new, int32_t head_dim, const void* dict_k, const void* dict_v,
                      int32_t n_atoms, uint32_t* k_lo, uint32_t* k_full, uint32_t* v_full,
                      int64_t cap, const int32_t* lens_host, void* workspace, size_t ws_bytes,
                      sdk_stream_t stream) {
  if (B < 1 || B > SDK_MAX_BATCH || Hkv < 1 || n_new < 0 || cap < 1) return SDK_ERR_INVALID_ARG;
  if (lens_host == nullptr || workspace == nullptr || !aligned(workspace, SDK_WS_ALIGN))
    return SDK_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return SDK_ERR_UNSUPPORTED;
  if (x_dtype != SDK_F32 && x_dtype != SDK_BF16) return SDK_ERR_INVALID_ARG;
  if (n_atoms < 1 || n_atoms > SDK_MAX_ATOMS) return SDK_ERR_INVALID_ARG;
  for (int b = 0; b < B; ++b) {
    if (lens_host[b] < 0) return SDK_ERR_INVALID_ARG;
    if ((int64_t)lens_host[b] + n_new > cap) return SDK_ERR_CAPACITY;
  }
  if (n_new == 0) return SDK_OK;
  if (!xk || !xv || !dict_k || !dict_v || !k_lo || !k_full || !v_full) return SDK_ERR_INVALID_ARG;
  if (!aligned(k_full, 16) || !aligned(v_full, 16) || !aligned(k_lo, 4)) return SDK_ERR_INVALID_ARG;
  if (ws_bytes < sdk_append_workspace_bytes(B, Hkv, n_new, head_dim, n_atoms))
    return SDK_ERR_CAPACITY;
  const int64_t nv = (int64_t)B * Hkv * n_new;
  char* ws = reinterpret_cast<char*>(workspace);
  const size_t hb = align_up(sizeof(WsHeader), 256);
  const size_t cb = align_up((size_t)nv * kAtoms * 4, 256);
  uint32_t* codes2[2] = {reinterpret_cast<uint32_t*>(ws + hb),
                         reinterpret_cast<uint32_t*>(ws + hb + cb)};
  char* scratch = ws + hb + 2 * cb;
  const size_t scratch_bytes = sdk_append_workspace_bytes(B, Hkv, n_new, head_dim, n_atoms) - hb - 2 * cb;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // a few vectors: the atom-parallel encoder writes straight into the store,
  // K and V in one launch when both fit
  if (nv <= kSmallEncodeRows) {
    SmallEncode e;
    memset(&e, 0, sizeof(e));
    for (int s = 0; s < 2; ++s) {
      EncodeParams& p = e.p[s];
      p.x = s == 0 ? xk : xv;
      p.x_dtype = x_dtype;
      p.n_vec = nv;
      p.dict = reinterpret_cast<const uint16_t*>(s == 0 ? dict_k : dict_v);
      p.n = n_atoms;
      p.k_atoms = kAtoms;
      p.codes = s == 0 ? k_full : v_full;
      p.rsq = nullptr;
      p.hdr = reinterpret_cast<WsHeader*>(ws);
    }
    e.head_dim = head_dim;
    e.append = true;
    e.lo[0] = k_lo;
    e.lo[1] = nullptr;
    e.cap = cap;
    e.B = B;
    e.Hkv = Hkv;
    e.n_new = n_new;
    e.lens = lens_host;
    e.rs = record_stride(k_full, v_full);
    e.streams = 2;
    bool taken = false;
    sdk_status rc = launch_encode_small(e, scratch, scratch_bytes, st, &taken);
    if (taken) return rc;
    SmallEncode one = e;
    one.streams = 1;
    rc = launch_encode_small(one, scratch, scratch_bytes, st, &taken);
    if (taken) {
      if (rc != SDK_OK) return rc;
      one.p[0] = e.p[1];
      one.lo[0] = nullptr;
      rc = launch_encode_small(one, scratch, scratch_bytes, st, &taken);
      if (!taken) return SDK_ERR_CUDA;  // the same shape was taken just before
      return rc;
    }
  }
  // K and V: one tensor-core launch over the row tiles of both streams
  // (or, where it does not apply, one encode per stream), then the words
  // go into the store
  EncodeParams pe[2];
  for (int s = 0; s < 2; ++s) {
    EncodeParams& p = pe[s];
    p.x = s == 0 ? xk : xv;
    p.x_dtype = x_dtype;
    p.n_vec = nv;
    p.dict = reinterpret_cast<const uint16_t*>(s == 0 ? dict_k : dict_v);
    p.n = n_atoms;
    p.k_atoms = kAtoms;
    p.codes = codes2[s];
    p.rsq = nullptr;
    p.hdr = reinterpret_cast<WsHeader*>(ws);
  }
  bool taken = false;
  sdk_status rc = launch_encode_tc(pe, 2, head_dim, scratch, scratch_bytes, st, &taken);
  if (rc != SDK_OK) return rc;
  for (int s = 0; s < 2 && !taken; ++s) {
    rc = encode_core(true, pe[s], head_dim, scratch, scratch_bytes, st);
    if (rc != SDK_OK) return rc;
  }
  for (int s = 0; s < 2; ++s) {
    ScatterParams sp;
    sp.codes = codes2[s];
    sp.full = s == 0 ? k_full : v_full;
    sp.lo = s == 0 ? k_lo : nullptr;
    sp.cap = cap;
    sp.Hkv = Hkv;
    sp.n_new = n_new;
    sp.rs = record_stride(k_full, v_full);
    sp.nv = nv;
    for (int b = 0; b < B; ++b) sp.lens[b] = lens_host[b];
    const int64_t tot = nv * kAtoms;
    scatter_codes_kernel<<<(unsigned)((tot + 255) / 256), 256, 0, st>>>(sp);
    if (cudaGetLastError() != cudaSuccess) return SDK_ERR_CUDA;
  }
  return SDK_OK;
}

}  // extern "C"

// ------------------------------------------------------------------ decode

extern "C" {

size_t sdk_decode_workspace_bytes(int32_t B, int32_t Hq, int32_t head_dim, int32_t n_atoms,
                                  int64_t max_len) {
  if (B < 1 || Hq < 1 || n_atoms < 1 || max_len < 1 || (head_dim != 64 && head_dim != 128))
    return 0;
  return decode_layout(B, Hq, head_dim, n_atoms, max_len).total;
}

sdk_status sdk_decode_layout_of(int32_t B, int32_t Hq, int32_t head_dim, int32_t n_atoms,
                                int64_t max_len, sdk_decode_layout* layout_out) {
  if (layout_out == nullptr || B < 1 || Hq < 1 || n_atoms < 1 || max_len < 1)
    return SDK_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return SDK_ERR_UNSUPPORTED;
  *layout_out = decode_layout(B, Hq, head_dim, n_atoms, max_len);
  return SDK_OK;
}

}  // extern "C"

// The default selection: radix histograms of all keys, unless
// SDK_DECODE_BRACKET=1 (read once per process) makes the sampled bracket
// the default.  Measured per 256K layer: radix 29.9 + 19.7 + 9.5 us
// (Klow scan, pass 2, final), bracket 22.8 + 43.4 + 14.7 us (sample,
// classifying Klow scan, select).
static bool bracket_selection() {
  static int on = -1;
  if (on < 0) {
    const char* v = getenv("SDK_DECODE_BRACKET");
    on = (v != nullptr && v[0] == '1') ? 1 : 0;
  }
  return on == 1;
}

// Checks the decode arguments and fills the kernel parameter block.  With
// glens (the sequences' whole lengths; context-sharded decode) the selected
// set size k comes from glens[b] and lens_host holds this rank's shard.
static sdk_status build_decode_params(const float* q, int32_t B, int32_t Hq, int32_t Hkv,
                                      int32_t head_dim, const void* dict_k, const void* dict_v,
                                      int32_t n_atoms, const uint32_t* k_lo,
                                      const uint32_t* k_full, const uint32_t* v_full, int64_t cap,
                                      const int32_t* lens_host, const int32_t* glens,
                                      int32_t klow, int32_t khigh, int32_t top_num,
                                      int32_t top_den, int32_t flags, float scale, float* out,
                                      void* workspace, size_t ws_bytes, DecodeParams& p) {
  if (B < 1 || B > SDK_MAX_BATCH || Hq < 1 || Hkv < 1 || Hq % Hkv != 0) return SDK_ERR_INVALID_ARG;
  if ((int64_t)B * Hq > 2048) return SDK_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return SDK_ERR_UNSUPPORTED;
  if (n_atoms < 1 || n_atoms > SDK_MAX_ATOMS || cap < 1) return SDK_ERR_INVALID_ARG;
  if (klow < 1 || khigh < klow || khigh > SDK_K_ATOMS) return SDK_ERR_INVALID_ARG;
  if (top_num < 1 || top_den < 1 || top_num > top_den) return SDK_ERR_INVALID_ARG;
  if (!(scale > 0.0f) || !std::isfinite(scale)) return SDK_ERR_INVALID_ARG;
  if (flags & ~(SDK_DECODE_FULL_SOFTMAX | SDK_DECODE_INT_SOFTMAX | SDK_DECODE_KEEP_KEYS |
                SDK_DECODE_SELECT_RADIX | SDK_DECODE_SELECT_BRACKET))
    return SDK_ERR_INVALID_ARG;
  if ((flags & SDK_DECODE_SELECT_RADIX) && (flags & SDK_DECODE_SELECT_BRACKET))
    return SDK_ERR_INVALID_ARG;
  if (!q || !dict_k || !dict_v || !k_lo || !k_full || !v_full || !out || !lens_host || !workspace)
    return SDK_ERR_INVALID_ARG;
  if (!aligned(workspace, SDK_WS_ALIGN) || !aligned(dict_k, 16) || !aligned(dict_v, 16) ||
      !aligned(k_full, 16) || !aligned(v_full, 16) || !aligned(k_lo, 4) || !aligned(q, 16) ||
      !aligned(out, 16))
    return SDK_ERR_INVALID_ARG;
  int64_t max_len = 0;
  for (int b = 0; b < B; ++b) {
    if (lens_host[b] < 1 || lens_host[b] > cap) return SDK_ERR_INVALID_ARG;
    if (glens != nullptr && glens[b] < lens_host[b]) return SDK_ERR_INVALID_ARG;
    if (lens_host[b] > max_len) max_len = lens_host[b];
  }
  const sdk_decode_layout l = decode_layout(B, Hq, head_dim, n_atoms, max_len);
  if (ws_bytes < l.total) return SDK_ERR_CAPACITY;

  std::memset(&p, 0, sizeof(p));
  char* ws = reinterpret_cast<char*>(workspace);
  p.q = q;
  p.dk = reinterpret_cast<const uint16_t*>(dict_k);
  p.dv = reinterpret_cast<const uint16_t*>(dict_v);
  p.k_lo = k_lo;
  p.k_full = k_full;
  p.v_full = v_full;
  p.out = out;
  p.hdr = reinterpret_cast<WsHeader*>(ws + l.header);
  p.qd = reinterpret_cast<float*>(ws + l.qd);
  p.keys = reinterpret_cast<uint32_t*>(ws + l.keys);
  p.hist1 = reinterpret_cast<uint32_t*>(ws + l.hist1);
  p.hist2 = reinterpret_cast<uint32_t*>(ws + l.hist2);
  p.st = reinterpret_cast<sdk_select_state*>(ws + l.state);
  p.list = reinterpret_cast<int32_t*>(ws + l.list);
  p.cand_t = reinterpret_cast<int32_t*>(ws + l.cand_t);
  p.cand_key = reinterpret_cast<uint32_t*>(ws + l.cand_key);
  p.sel_score = reinterpret_cast<float*>(ws + l.sel_score);
  p.w = reinterpret_cast<uint16_t*>(ws + l.w);
  p.part = reinterpret_cast<float*>(ws + l.part);
  p.cap = cap;
  p.L = (int64_t)l.row;   // row stride of the per-token regions
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.g = Hq / Hkv;
  p.d = head_dim;
  p.n = n_atoms;
  p.klow = klow;
  p.khigh = khigh;
  p.full = (flags & SDK_DECODE_FULL_SOFTMAX) ? 1 : 0;
  p.isoft = (flags & SDK_DECODE_INT_SOFTMAX) ? 1 : 0;
  // the sampled-bracket selection unless the softmax runs over every token
  // (that path needs every key and the complement list) or
  // SDK_DECODE_BRACKET=0 is set in the environment
  const bool want_bracket = (flags & SDK_DECODE_SELECT_BRACKET) ? true
                            : (flags & SDK_DECODE_SELECT_RADIX) ? false
                                                                : bracket_selection();
  p.bracket = (!p.full && want_bracket) ? 1 : 0;
  p.keep_keys = (flags & SDK_DECODE_KEEP_KEYS) ? 1 : 0;
  p.rs = record_stride(k_full, v_full);
  p.R = B * Hq;
  p.n_out_tiles = (n_atoms + 127) / 128;
  p.scale = scale;
  p.world = 1;
  p.tok_off[0] = p.sel_off[0] = p.dom_off[0] = 0;
  for (int b = 0; b < B; ++b) {
    const int64_t N = lens_host[b];
    const int64_t G = glens != nullptr ? glens[b] : N;
    int64_t k = ((int64_t)top_num * G + top_den - 1) / top_den;
    if (k < 1) k = 1;
    if (k > G) k = G;
    p.lens[b] = (int)N;
    p.kcnt[b] = (int)k;
    p.dcnt[b] = p.full ? (int)N : (int)k;
    p.tok_off[b + 1] = p.tok_off[b] + (int64_t)Hq * N;
    p.sel_off[b + 1] = p.sel_off[b] + (int64_t)Hq * k;
    p.dom_off[b + 1] = p.dom_off[b] + (int64_t)Hq * p.dcnt[b];
  }
  return SDK_OK;
}

extern "C" {

sdk_status sdk_decode_attn(const float* q, int32_t B, int32_t Hq, int32_t Hkv, int32_t head_dim,
                           const void* dict_k, const void* dict_v, int32_t n_atoms,
                           const uint32_t* k_lo, const uint32_t* k_full, const uint32_t* v_full,
                           int64_t cap, const int32_t* lens_host, int32_t klow, int32_t khigh,
                           int32_t top_num, int32_t top_den, int32_t flags, float scale,
                           float* out, void* workspace, size_t ws_bytes, sdk_stream_t stream) {
  DecodeParams p;
  const sdk_status s = build_decode_params(q, B, Hq, Hkv, head_dim, dict_k, dict_v, n_atoms, k_lo,
                                           k_full, v_full, cap, lens_host, nullptr, klow, khigh,
                                           top_num, top_den, flags, scale, out, workspace,
                                           ws_bytes, p);
  if (s != SDK_OK) return s;
  return launch_decode(p, reinterpret_cast<cudaStream_t>(stream));
}

sdk_status sdk_decode_attn_shard(int32_t stage, int32_t rank, int32_t world, const void* gathered,
                                 const float* q, int32_t B, int32_t Hq, int32_t Hkv,
                                 int32_t head_dim, const void* dict_k, const void* dict_v,
                                 int32_t n_atoms, const uint32_t* k_lo, const uint32_t* k_full,
                                 const uint32_t* v_full, int64_t cap, const int32_t* lens_host,
                                 const int32_t* glens_host, int32_t klow, int32_t khigh,
                                 int32_t top_num, int32_t top_den, int32_t flags, float scale,
                                 float* out, void* workspace, size_t ws_bytes,
                                 sdk_stream_t stream) {
  if (stage < 1 || stage > 6 || world < 1 || rank < 0 || rank >= world) return SDK_ERR_INVALID_ARG;
  if (flags != 0) return SDK_ERR_UNSUPPORTED;   // selected-set fp32 softmax only
  if (glens_host == nullptr) return SDK_ERR_INVALID_ARG;
  if ((stage == 5 || stage == 6) && (gathered == nullptr || !aligned(gathered, 8)))
    return SDK_ERR_INVALID_ARG;
  DecodeParams p;
  const sdk_status s = build_decode_params(q, B, Hq, Hkv, head_dim, dict_k, dict_v, n_atoms, k_lo,
                                           k_full, v_full, cap, lens_host, glens_host, klow, khigh,
                                           top_num, top_den, flags, scale, out, workspace,
                                           ws_bytes, p);
  if (s != SDK_OK) return s;
  p.world = world;
  p.shard_in = gathered;
  p.bracket = 0;   // the context-sharded stages exchange radix histograms
  return launch_decode(p, reinterpret_cast<cudaStream_t>(stream), stage, rank);
}

sdk_status sdk_timing_enable(int32_t on) { return timing_enable(on != 0); }

int32_t sdk_timing_read(float* ms_out, int32_t max_n) { return timing_read(ms_out, max_n); }

sdk_status sdk_workspace_init(void* workspace, size_t ws_bytes, sdk_stream_t stream) {
  if (workspace == nullptr || !aligned(workspace, SDK_WS_ALIGN) || ws_bytes < sizeof(WsHeader))
    return SDK_ERR_INVALID_ARG;
  return cudaMemsetAsync(workspace, 0, sizeof(WsHeader), reinterpret_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? SDK_OK
             : SDK_ERR_CUDA;
}

sdk_status sdk_check_status(void* workspace, sdk_stream_t stream, uint32_t* counters_out) {
  if (workspace == nullptr || !aligned(workspace, SDK_WS_ALIGN)) return SDK_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  uint32_t h[4] = {0, 0, 0, 0};
  if (cudaStreamSynchronize(st) != cudaSuccess) return SDK_ERR_CUDA;
  if (cudaMemcpy(h, workspace, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess)
    return SDK_ERR_CUDA;
  if (counters_out) std::memcpy(counters_out, h, sizeof(h));
  if (h[0] != 0u) {
    const uint32_t zero[2] = {0u, 0u};
    if (cudaMemcpy(workspace, zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess)
      return SDK_ERR_CUDA;
  }
  return (sdk_status)h[0];
}

}  // extern "C"
