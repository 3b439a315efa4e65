// Internal helpers shared by the kernels of libsdk.so (not installed).
//
// Code word format (review of "LLM Inference in a Flash!", FAQ on the 15x
// KV compression: each vector is stored as the indices and coefficients of
// its 16 atoms): bits 31..16 = fp16 coefficient, bit 15 = 0, bits 14..0 =
// atom index.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "../../include/sdk.h"

namespace sdk {

constexpr int kMaxAtoms = SDK_MAX_ATOMS;
constexpr int kAtoms = SDK_K_ATOMS;
constexpr int kLoPlanes = SDK_KLOW_PLANES;
constexpr int kMaxBatch = SDK_MAX_BATCH;

// Header at offset 0 of every workspace (256 bytes).
struct WsHeader {
  unsigned int err;          // first recorded sdk_status (0 = none)
  unsigned int info;         // detail of that failure
  unsigned int enc_fallback; // encode rows re-scanned exactly
  unsigned int enc_cands;    // encode candidates re-scored in fp32
  unsigned int pad[60];
};
static_assert(sizeof(WsHeader) == 256, "header size");

__device__ __forceinline__ void record_error(WsHeader* h, unsigned code,
                                             unsigned info) {
  if (atomicCAS(&h->err, 0u, code) == 0u) atomicExch(&h->info, info);
}

// ---- code words -----------------------------------------------------------
__device__ __forceinline__ uint32_t word_idx(uint32_t w) { return w & 0x7FFFu; }
__device__ __forceinline__ float word_coef(uint32_t w) {
  return __half2float(__ushort_as_half((unsigned short)(w >> 16)));
}
// fp16 round-to-nearest-even with saturation to +-65504.
__device__ __forceinline__ uint32_t make_word(float coef, uint32_t idx) {
  float c = fminf(fmaxf(coef, -65504.0f), 65504.0f);
  uint32_t hb = (uint32_t)__half_as_ushort(__float2half_rn(c));
  return (hb << 16) | (idx & 0x7FFFu);
}

// ---- order-preserving float keys -------------------------------------------
// Larger key <=> larger score; -0 and +0 share the key of +0.
__device__ __forceinline__ uint32_t score_key(float s) {
  uint32_t b = __float_as_uint(s);
  if ((b << 1) == 0u) b = 0u;  // -0 -> +0
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float key_score(uint32_t k) {
  uint32_t b = (k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k;
  return __uint_as_float(b);
}

// Chris Wellons' "lowbias32" integer hash (from his 2018 search for 32-bit
// hash functions with low bias): picks the sampled token of each block in
// the sampled-bracket selection.
__host__ __device__ __forceinline__ uint32_t lowbias32(uint32_t x) {
  x ^= x >> 16;
  x *= 0x7feb352dU;
  x ^= x >> 15;
  x *= 0x846ca68bU;
  x ^= x >> 16;
  return x;
}

__device__ __forceinline__ float bf16_lo(uint32_t v) {
  return __uint_as_float(v << 16);
}
__device__ __forceinline__ float bf16_hi(uint32_t v) {
  return __uint_as_float(v & 0xFFFF0000u);
}

// ---- block-wide helpers (blockDim.x a multiple of 32, <= 1024) -------------
// Inclusive scan of one uint32 per thread; returns the block total in *total.
__device__ __forceinline__ uint32_t block_incl_scan(uint32_t v, uint32_t* s_warp,
                                                    uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nw = blockDim.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t t = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += t;
  }
  __syncthreads();
  if (lane == 31) s_warp[warp] = v;
  __syncthreads();
  if (warp == 0) {
    uint32_t t = lane < nw ? s_warp[lane] : 0u;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      uint32_t u = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += u;
    }
    if (lane < nw) s_warp[lane] = t;
  }
  __syncthreads();
  uint32_t base = warp > 0 ? s_warp[warp - 1] : 0u;
  *total = s_warp[nw - 1];
  __syncthreads();
  return base + v;
}

// Programmatic dependent launch: a kernel launched with programmatic stream
// serialization may start while the previous kernel of the stream drains;
// pdl_wait() blocks until that kernel has completed and its memory is
// visible (a no-op for an ordinary launch).  pdl_launch() lets the next
// kernel of the stream start launching.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// 16-byte asynchronous global -> shared copy (L2 only, no registers); with
// valid == false nothing is read and the 16 bytes are zero-filled (the
// source operand is then only a placeholder address).
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc, bool valid) {
  const unsigned d = (unsigned)__cvta_generic_to_shared(smem_dst);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(gsrc),
               "r"(valid ? 16 : 0)
               : "memory");
}
// The same with the L2 fetch widened to the whole 128-byte line (for a
// record whose line holds data needed later).
__device__ __forceinline__ void cp_async16_128B(void* smem_dst, const void* gsrc, bool valid) {
  const unsigned d = (unsigned)__cvta_generic_to_shared(smem_dst);
  asm volatile("cp.async.cg.shared.global.L2::128B [%0], [%1], 16, %2;" ::"r"(d), "l"(gsrc),
               "r"(valid ? 16 : 0)
               : "memory");
}
// The same under an L2 eviction policy (createpolicy), fetching the whole
// 128-byte line.
__device__ __forceinline__ void cp_async16_128B_pol(void* smem_dst, const void* gsrc, bool valid,
                                                    uint64_t pol) {
  const unsigned d = (unsigned)__cvta_generic_to_shared(smem_dst);
  asm volatile("cp.async.cg.shared.global.L2::cache_hint.L2::128B [%0], [%1], 16, %2, %3;" ::"r"(d),
               "l"(gsrc), "r"(valid ? 16 : 0), "l"(pol)
               : "memory");
}
// The same with the L2 prefetch size limited to 64 bytes (for 64-byte
// records at scattered addresses).
__device__ __forceinline__ void cp_async16_64B(void* smem_dst, const void* gsrc, bool valid) {
  const unsigned d = (unsigned)__cvta_generic_to_shared(smem_dst);
  asm volatile("cp.async.cg.shared.global.L2::64B [%0], [%1], 16, %2;" ::"r"(d), "l"(gsrc),
               "r"(valid ? 16 : 0)
               : "memory");
}
// 16-byte copy of which only the first `bytes` (0..16) are read; the rest
// of the 16 destination bytes is zero-filled.
__device__ __forceinline__ void cp_async16_n(void* smem_dst, const void* gsrc, unsigned bytes) {
  const unsigned d = (unsigned)__cvta_generic_to_shared(smem_dst);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(gsrc), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
// waits until at most N of this thread's committed groups are in flight
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ uint32_t warp_umax(uint32_t v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}


// ---- kernel parameter blocks (passed by value) ------------------------------
// Decode: one layer, B sequences, R = B*Hq query heads.  Per sequence b:
// lens = tokens, kcnt = selected-set size, dcnt = softmax-domain size;
// *_off = prefix sums over sequences of Hq * (that count).
struct DecodeParams {
  const float* q;
  const uint16_t* dk;
  const uint16_t* dv;
  const uint32_t* k_lo;
  const uint32_t* k_full;
  const uint32_t* v_full;
  float* out;
  float* qd;
  uint32_t* keys;
  uint32_t* hist1;
  uint32_t* hist2;
  sdk_select_state* st;
  int32_t* list;
  int32_t* cand_t;
  uint32_t* cand_key;
  float* sel_score;
  uint16_t* w;           // bf16 [3][R][n]: w = w[0] + w[1] + w[2] per (row, atom)
  float* part;
  WsHeader* hdr;
  int64_t cap;
  int64_t L;
  int B, Hq, Hkv, g, d, n, klow, khigh, full, isoft, R, n_out_tiles;
  // selection by a sampled bracket of the k-th key (sample_kernel,
  // klow_kernel<1>, select_kernel) instead of radix histograms; keep_keys:
  // the Klow scan also stores every token's key (SDK_DECODE_KEEP_KEYS)
  int bracket, keep_keys;
  // words between consecutive tokens' records in k_full / v_full: 16, or
  // 32 when the two point into one interleaved array [..][cap][2][16]
  // (v_full = k_full + 16: a token's key and value records form one
  // 128-byte line)
  int rs;
  int klow_buf;          // bracket-path Klow scan: buffer entries (selected; candidates half)
  // context-sharded decode: 0 = whole decode; 1 / 2 = attend's first /
  // second half (shard_in: the gathered softmax statistics); world ranks
  int att_mode, world;
  const void* shard_in;
  float scale;
  int lens[kMaxBatch];
  int kcnt[kMaxBatch];
  int dcnt[kMaxBatch];
  int64_t tok_off[kMaxBatch + 1];
  int64_t sel_off[kMaxBatch + 1];
  int64_t dom_off[kMaxBatch + 1];
};

// Encode: n_vec vectors of head_dim over n dictionary atoms, k_atoms picks.
struct EncodeParams {
  const void* x;
  int x_dtype;
  int64_t n_vec;
  const uint16_t* dict;
  int n;
  int k_atoms;
  uint32_t* codes;
  float* rsq;
  WsHeader* hdr;
};

int num_sms();  // cached multiprocessor count of the current device

// Limit of the waits for other CTAs' results (sdk_set_exchange_timeout_ns;
// 1 s by default); set_exchange_wait_ns returns the previous limit.
unsigned long long exchange_wait_ns();
unsigned long long set_exchange_wait_ns(unsigned long long ns);

// Kernel attributes (the dynamic shared-memory limits) are set per device:
// device_needs_setup tells whether the current device's bit in `flags` is
// still clear, device_setup_done sets it once the attributes are set.
// Concurrent first calls may both set the attributes, which is harmless;
// none launches before its own setup is complete.
bool device_needs_setup(const unsigned long long* flags);
void device_setup_done(unsigned long long* flags);

// QD on the tensor cores (taken = false: not available, use the CUDA cores)
sdk_status launch_qd_tc(const DecodeParams& p, cudaStream_t stream, bool* taken);
// out += w D_V on the tensor cores (taken = false: use the CUDA cores)
sdk_status launch_out_tc(const DecodeParams& p, cudaStream_t stream, bool* taken);
// shard_stage 0: the whole decode; 1..6: one stage of the context-sharded
// decode for rank rank_id (sdk_decode_attn_shard)
sdk_status launch_decode(DecodeParams p, cudaStream_t stream, int shard_stage = 0,
                         int rank_id = 0);
// kernel timing (sdk_timing_enable / sdk_timing_read): the next slot's
// event pair (nulls when timing is off) and a record that also works inside
// a stream capture
sdk_status timing_enable(bool on);
int timing_read(float* ms_out, int max_n);
void timing_slot(cudaEvent_t* e0, cudaEvent_t* e1);
cudaError_t timing_record(cudaEvent_t e, cudaStream_t stream);
sdk_decode_layout decode_layout(int B, int Hq, int d, int n, int64_t L);
sdk_status launch_encode_simt(const EncodeParams& p, int head_dim, cudaStream_t stream);
// Tensor-core encoder of one or two streams (ps[0..streams-1]; two
// streams need equal n, k_atoms and x_dtype) in one launch; sets *taken =
// false when it does not handle the shape (the caller then runs the
// CUDA-core encoder).
sdk_status launch_encode_tc(const EncodeParams* ps, int streams, int head_dim, void* scratch,
                            size_t scratch_bytes, cudaStream_t stream, bool* taken);
// scratch of launch_encode_tc for n_vec vectors in all over `streams` streams
size_t encode_tc_scratch_bytes(int64_t n_vec, int head_dim, int n_atoms, int streams = 1);

// Atom-parallel encoder for a few vectors of one or two streams (rows per
// call: 64 in total, the second stream starting at an even slot).  In
// append mode p[s].codes is the code store (full words) and lo[s] the
// first-3 planes (or null); words land at token lens[b] + i.
struct SmallEncode {
  EncodeParams p[2];
  int streams;
  int head_dim;
  bool append;
  uint32_t* lo[2];
  int64_t cap;
  int B, Hkv, n_new;
  int rs;               // words between tokens' records in the store (16 or 32)
  const int32_t* lens;  // host, [B]
};
// Sets *taken = false when it does not handle the call (too many rows,
// dictionary too large for one wave, switched off by SDK_ENCODE_SMALL=0).
sdk_status launch_encode_small(const SmallEncode& e, void* scratch, size_t scratch_bytes,
                               cudaStream_t stream, bool* taken);
size_t encode_small_scratch_bytes();
constexpr int64_t kSmallEncodeRows = 64;

}  // namespace sdk
