/*
 * sdk.h -- dictionary-coded KV cache, encode and decode-attention hot path
 *          for NVIDIA B200 (sm_100a).  C ABI of libsdk.so.
 *
 * Method: "LLM Inference in a Flash!" (Zhao, Kim, Hooper, Manolache, Mahoney,
 * Shao, Keutzer, Gholami).  The evolve.pub review of the paper, section
 * "Summary", and its FAQ entry "What is the 15x KV cache compression ..."
 * describe what is computed here:
 *   - every key and value vector is stored as K=16 (atom index, coefficient)
 *     pairs over a static, per-layer, per-stream (key or value) overcomplete
 *     dictionary of 32,768 atoms;
 *   - the encoder is a projection-based greedy pursuit replacing OMP, so no
 *     least-squares refit is done;
 *   - decoding uses query-aware hierarchical sparsity: every token is scored
 *     from Klow=3 atoms, the top 10% are refined with Khigh=16 atoms.
 * The authors' abstract (readsearch.ai listing) states the goal: represent
 * each KV vector as a linear combination of static dictionary vectors.
 *
 * Conventions for every entry point
 *   - Pointers marked "device" are CUDA device pointers (or managed memory)
 *     owned by the caller; pointers marked "host" are host memory read
 *     during the call only.  The library allocates nothing.
 *   - Calls are stream-ordered and asynchronous on `stream` (NULL = the
 *     legacy default stream).  Host-side argument checks return an error
 *     BEFORE anything is launched; a launch failure returns SDK_ERR_CUDA.
 *   - Conditions found on the device (an atom index >= n_atoms, an
 *     inconsistent selection count) are recorded in the workspace header and
 *     read by sdk_check_status(); no kernel traps.
 *   - Thread safety: concurrent calls must use distinct workspaces.
 *   - Tensors are dense, row-major, with no padding between rows.
 *
 * Code word (32 bits): bits 31..16 = fp16 bits of the coefficient (round to
 * nearest even, saturated to +-65504), bit 15 = 0, bits 14..0 = atom index.
 *
 * Code store of one layer (capacity `cap` tokens per sequence):
 *   k_lo   uint32 [B][Hkv][3][cap]  words 0..2 (greedy order) of every key
 *                                   code, one plane per word: the Klow scan
 *                                   reads 12 bytes per token, coalesced.
 *   k_full uint32 [B][Hkv][cap][16] all 16 words of every key code: one
 *                                   64-byte record per token for the
 *                                   Khigh rescore of selected tokens.
 *   v_full uint32 [B][Hkv][cap][16] all 16 words of every value code.
 * Query head h of a sequence reads KV head h / (Hq / Hkv).
 */
#ifndef SDK_H
#define SDK_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define SDK_API __attribute__((visibility("default")))
#else
#define SDK_API
#endif

/* A cudaStream_t, declared without including the CUDA headers. */
typedef struct CUstream_st* sdk_stream_t;

typedef enum {
  SDK_OK = 0,
  SDK_ERR_INVALID_ARG = 1,   /* null pointer, bad size, misaligned buffer */
  SDK_ERR_UNSUPPORTED = 2,   /* valid but outside what is built (head_dim) */
  SDK_ERR_CAPACITY = 3,      /* append past `cap`, workspace too small     */
  SDK_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed       */
  SDK_ERR_TIMEOUT = 5,       /* a bounded device wait gave up              */
  SDK_ERR_DEVICE_CHECK = 6   /* a device-side check failed (bad atom index) */
} sdk_status;

typedef enum { SDK_F32 = 0, SDK_BF16 = 1 } sdk_dtype;

#define SDK_MAX_ATOMS 32768   /* 15-bit atom index                         */
#define SDK_K_ATOMS 16        /* atoms per stored code                     */
#define SDK_KLOW_PLANES 3     /* words kept in the k_lo planes             */
#define SDK_MAX_BATCH 64      /* sequences per decode / append call        */
#define SDK_WS_ALIGN 256      /* required alignment of workspaces (bytes)  */

/* Human-readable name of a status code (static string, never NULL). */
SDK_API const char* sdk_status_string(int status);

/* Library ABI version (incremented on any signature change). */
SDK_API int32_t sdk_version(void);

/* Limit, in nanoseconds of the GPU's global timer, of every device-side
 * wait for another CTA's result: the small-batch encoder's per-step
 * exchange of slice winners (sdk_encode / sdk_append with at most 64
 * vectors).  A wait that runs out records SDK_ERR_TIMEOUT in the
 * workspace header (read by sdk_check_status); the kernel then leaves its
 * loop, frees its tensor memory and returns, and the CTAs waiting for it
 * run out in turn.  No copy or MMA of the CTA is in flight at these waits.
 * Process-wide; default 1 s; 0 gives up at the first word that is not
 * there yet.  Returns the previous limit.  The waits on the CTA's own
 * copies and MMAs (mbarriers) keep their fixed 1 s limit.  The paper has
 * no counterpart: this is the failure detection of the device waits. */
SDK_API uint64_t sdk_set_exchange_timeout_ns(uint64_t ns);

/* ------------------------------------------------------------------ encode
 * Greedy pursuit ("LLM Inference in a Flash!", review Summary): for every
 * input vector x, r = x; 16 times: i* = argmax_i |<r, d_i>| (ties: lowest
 * i), coef = <r, d_i*>, r -= coef * d_i*.  The pick is made exactly in
 * fp32: candidate atoms come from a bf16 tensor-core correlation GEMM with
 * fp32 accumulation, and every atom that can be the fp32 argmax within the
 * rounding bound of that GEMM is re-scored in fp32 before the pick.
 *
 *   x           device, [n_vec][head_dim], fp32 or bf16 (x_dtype)
 *   n_vec       number of vectors, >= 0 (0 launches nothing)
 *   head_dim    64 or 128
 *   dict        device, bf16 [n_atoms][head_dim], unit-norm rows expected
 *               (used as given), 16-byte aligned
 *   n_atoms     1 .. 32768
 *   k_atoms     1 .. 16 picks per vector
 *   codes_out   device, uint32 [n_vec][k_atoms], words in pick order
 *   resid_sqnorm_out  device, float [n_vec] = ||r_final||^2, or NULL
 *   workspace   device, >= sdk_encode_workspace_bytes(), 256-byte aligned,
 *               initialised once by sdk_workspace_init()
 * Errors: SDK_ERR_INVALID_ARG (null/misaligned pointers, sizes out of
 * range), SDK_ERR_UNSUPPORTED (head_dim), SDK_ERR_CAPACITY (ws_bytes too
 * small), SDK_ERR_CUDA.
 */
SDK_API sdk_status sdk_encode(const void* x, int32_t x_dtype, int64_t n_vec,
                      int32_t head_dim, const void* dict, int32_t n_atoms,
                      int32_t k_atoms, uint32_t* codes_out,
                      float* resid_sqnorm_out, void* workspace,
                      size_t ws_bytes, sdk_stream_t stream);

/* Same contract as sdk_encode, computed by the plain CUDA-core kernel:
 * every correlation in fp32 FMA order k = 0..head_dim-1, exact argmax over
 * all atoms.  A second, independent GPU path for cross-checks and for
 * head_dim / n_atoms the tensor-core kernel does not take. */
SDK_API sdk_status sdk_encode_simt(const void* x, int32_t x_dtype, int64_t n_vec,
                           int32_t head_dim, const void* dict,
                           int32_t n_atoms, int32_t k_atoms,
                           uint32_t* codes_out, float* resid_sqnorm_out,
                           void* workspace, size_t ws_bytes,
                           sdk_stream_t stream);

SDK_API size_t sdk_encode_workspace_bytes(int64_t n_vec, int32_t head_dim,
                                  int32_t n_atoms);

/* ------------------------------------------------------------------ append
 * Encode n_new new key and value vectors per (sequence, KV head) and write
 * them into the code store at token positions [lens[b], lens[b] + n_new).
 * The review's FAQ describes the store: compact per-token codes referencing
 * a fixed dictionary, appended at every generated token while the
 * dictionary stays static.
 *
 *   xk, xv      device, [B][Hkv][n_new][head_dim], fp32 or bf16
 *   dict_k/_v   device, bf16 [n_atoms][head_dim]
 *   k_lo, k_full, v_full  device, the code store (layout above)
 *   cap         capacity in tokens per sequence
 *   lens_host   host, int32 [B]: current lengths; lens[b] + n_new <= cap.
 *               The library does not update it.
 * Errors: as sdk_encode, plus SDK_ERR_CAPACITY when lens[b] + n_new > cap.
 */
SDK_API sdk_status sdk_append(const void* xk, const void* xv, int32_t x_dtype,
                      int32_t B, int32_t Hkv, int32_t n_new, int32_t head_dim,
                      const void* dict_k, const void* dict_v, int32_t n_atoms,
                      uint32_t* k_lo, uint32_t* k_full, uint32_t* v_full,
                      int64_t cap, const int32_t* lens_host, void* workspace,
                      size_t ws_bytes, sdk_stream_t stream);

SDK_API size_t sdk_append_workspace_bytes(int32_t B, int32_t Hkv, int32_t n_new,
                                  int32_t head_dim, int32_t n_atoms);

/* decode flags */
#define SDK_DECODE_FULL_SOFTMAX 1   /* softmax over every token, not only S   */
#define SDK_DECODE_INT_SOFTMAX 2    /* integer softmax (see sdk_decode_attn)  */
#define SDK_DECODE_KEEP_KEYS 4      /* also store every token's s_lo key in
                                       the workspace region `keys` (for
                                       inspection; costs 4 B per token and
                                       query head of extra writes)           */
#define SDK_DECODE_SELECT_RADIX 8   /* find the top-k set by radix histograms
                                       of all keys                           */
#define SDK_DECODE_SELECT_BRACKET 16 /* find it through a sampled bracket of
                                       the k-th key (ignored with
                                       SDK_DECODE_FULL_SOFTMAX); without
                                       either flag the library's default     */

/* ------------------------------------------------------------ decode attn
 * One layer of decode attention for B sequences over their code stores
 * (review Summary: score all tokens at Klow=3, refine the top 10% at
 * Khigh=16).  Per query head (b, h), with N = lens[b]:
 *   QD      = D_K q                       (all n_atoms correlations)
 *   s_lo_t  = sum_{j<klow} c_tj QD[idx_tj]           for every token t
 *   S       = the k = ceil(top_num*N/top_den) tokens with the largest s_lo
 *             (ties: lower token index)
 *   s_t     = scale * sum_{j<khigh} c_tj QD[idx_tj]  for t in S
 *   p       = softmax of s over S; with flags & SDK_DECODE_FULL_SOFTMAX the
 *             softmax runs over all N tokens, t outside S using
 *             scale * s_lo_t.  With flags & SDK_DECODE_INT_SOFTMAX the
 *             softmax is integer (review Summary: integer polynomial
 *             Softmax on token-wise INT16 requantised inputs, bit-shift
 *             guards against INT32 overflow, fixed-point reciprocals):
 *             the head's fp32 logits l are requantised to q = rint(l / S),
 *             S = max|l| / 32767; e = I-BERT's integer exponential of
 *             (q - max q) >> sh (second-order polynomial on (-ln 2, 0] and
 *             a shift by the whole multiples of ln 2; sh the smallest shift
 *             keeping its squares below 2^31); P = (e * floor(2^61 / sum e))
 *             >> 31, probabilities in Q30.  `state` records sum e and sh.
 *   w[a]    = sum_t p_t sum_j c^V_tj [idx^V_tj == a] (over the softmax domain)
 *   out     = w D_V
 *
 *   q          device, float [B][Hq][head_dim], 16-byte aligned
 *   dict_k/_v  device, bf16 [n_atoms][head_dim]
 *   lens_host  host, int32 [B], 1 <= lens[b] <= cap
 *   klow       1 .. khigh;  khigh  klow .. 16
 *   top_num, top_den   0 < top_num <= top_den
 *   flags      0, or a combination of SDK_DECODE_FULL_SOFTMAX and
 *              SDK_DECODE_INT_SOFTMAX (other bits: SDK_ERR_INVALID_ARG)
 *   scale      logit scale (1/sqrt(head_dim) for standard attention)
 *   out        device, float [B][Hq][head_dim], 16-byte aligned
 *   workspace  device, >= sdk_decode_workspace_bytes(B, Hq, head_dim,
 *              n_atoms, max_len) with max_len >= every lens[b]
 * Limits: B <= 64, Hq % Hkv == 0, head_dim in {64, 128}, B*Hq <= 2048,
 *         scale > 0.
 * Selection (how S is found; the set is exact either way): by default
 * (and always with SDK_DECODE_FULL_SOFTMAX) a radix select over the keys
 * of all tokens (histograms of their digits).  With
 * SDK_DECODE_SELECT_BRACKET (or SDK_DECODE_BRACKET=1 in the environment
 * as the default), a sample of every head's tokens is scored first
 * and two of its order statistics bracket the k-th key; the Klow scan then
 * selects the tokens above the bracket and keeps those inside it as
 * candidates, among which the exact k-th key and the tie cut are found; a
 * head whose k-th key falls outside the bracket is re-scanned exactly
 * (state `select_path` 2).  The sample of KV head (b, kvh) with N tokens:
 * every token when N <= 8192; else, with blk = 8 * ceil(ceil(N / 1024) / 8)
 * and seed = lowbias32(0x9E3779B9 * (b * Hkv + kvh + 1)) (32-bit
 * arithmetic; lowbias32 is Chris Wellons' integer hash x ^= x >> 16,
 * x *= 0x7feb352d, x ^= x >> 15, x *= 0x846ca68b, x ^= x >> 16), block i
 * of blk tokens (len_i = min(blk, N - i * blk)) contributes the 8 tokens
 * from i * blk + 8 * (lowbias32(seed ^ i) mod (len_i / 8)), or all of its
 * tokens when len_i < 8.  The bracket is the sample's order statistics
 * 6 standard deviations of the sample rank above and below S * k / N.
 * Code store layout: k_full and v_full may also point into ONE array
 * uint32 [B][Hkv][cap][2][16] with v_full = k_full + 16 (a token's key and
 * value records adjacent in one 128-byte line); the library detects this
 * from the two pointers (here and in sdk_append).
 */
SDK_API sdk_status sdk_decode_attn(const float* q, int32_t B, int32_t Hq, int32_t Hkv,
                           int32_t head_dim, const void* dict_k,
                           const void* dict_v, int32_t n_atoms,
                           const uint32_t* k_lo, const uint32_t* k_full,
                           const uint32_t* v_full, int64_t cap,
                           const int32_t* lens_host, int32_t klow,
                           int32_t khigh, int32_t top_num, int32_t top_den,
                           int32_t flags, float scale, float* out,
                           void* workspace, size_t ws_bytes,
                           sdk_stream_t stream);

SDK_API size_t sdk_decode_workspace_bytes(int32_t B, int32_t Hq, int32_t head_dim,
                                  int32_t n_atoms, int64_t max_len);

/* ----------------------------------------- context-sharded decode attn
 * The same computation as sdk_decode_attn (flags 0: fp32 softmax over the
 * selected set) when every sequence's context is split over `world` ranks,
 * rank r holding a contiguous token range (ranks in token order, every
 * rank at least one token of every sequence).  Each rank runs stages 1..6
 * in order on its own shard and workspace; between stages the ranks
 * combine workspace regions (byte offsets from sdk_decode_layout_of for the
 * rank's own lens; R = B*Hq):
 *   after 1: sum over ranks, uint32 [R][4096] at `hist1` (the first-digit
 *            histograms of the keys);
 *   after 2: sum, uint32 [R][4096] at `hist2` (second digit, in the bucket);
 *   after 3: sum, uint32 [R][256] at `hist1` (third digit);
 *   after 4: all-gather the uint32 [R] at `hist2` (each rank's ties of the
 *            k-th key) into a device array [world][R], passed to stage 5;
 *   after 5: all-gather the float [R][2] at `hist2` + 4R bytes (each rank's
 *            largest logit and sum of exp(logit - largest) per head) into a
 *            device array [world][R][2], passed to stage 6;
 *   after 6: sum `out` over ranks.
 * The selected set is the exact global top k (k from glens, ties to the
 * lower global token index); the result equals sdk_decode_attn over the
 * whole context up to the order of fp32 additions.
 *   stage      1 .. 6
 *   rank, world   this rank, number of ranks
 *   gathered   device: stage 5 the [world][R] tie counts, stage 6 the
 *              [world][R][2] statistics (8-byte aligned); NULL otherwise
 *   lens_host  host, int32 [B], this rank's tokens of each sequence (>= 1);
 *              the code store holds them at positions 0 .. lens[b]-1
 *   glens_host host, int32 [B], every sequence's whole length
 *   others     as sdk_decode_attn; flags must be 0 (SDK_ERR_UNSUPPORTED)
 * The paper has no multi-device design; this follows the exchange the
 * decomposition of the selection and of the softmax needs.
 */
SDK_API sdk_status sdk_decode_attn_shard(int32_t stage, int32_t rank, int32_t world,
                           const void* gathered, const float* q, int32_t B,
                           int32_t Hq, int32_t Hkv, int32_t head_dim,
                           const void* dict_k, const void* dict_v,
                           int32_t n_atoms, const uint32_t* k_lo,
                           const uint32_t* k_full, const uint32_t* v_full,
                           int64_t cap, const int32_t* lens_host,
                           const int32_t* glens_host, int32_t klow,
                           int32_t khigh, int32_t top_num, int32_t top_den,
                           int32_t flags, float scale, float* out,
                           void* workspace, size_t ws_bytes,
                           sdk_stream_t stream);

/* ------------------------------------------------- decode, no workspace
 * sdk_decode_attn_static -- sdk_decode_attn with its workspace in a fixed
 * array of SDK_DECODE_STATIC_WS_BYTES (16 MiB) of the library's own device
 * memory, one per device, so that the call allocates nothing and takes no
 * workspace.  The paper has no counterpart: this is a calling convention
 * for hosts that cannot allocate device memory where they decode (a
 * serving loop whose memory is budgeted before the first request, a plain
 * C host without a device allocator of its own).
 *
 *   arguments  as sdk_decode_attn, without workspace/ws_bytes;
 *   status_out device, uint32 [2], 4-byte aligned, nullable: after the
 *              decode, the call copies in the first device-side failure
 *              recorded since the last such copy (status, detail; {0, 0} if
 *              none) and zeroes it in the array.  With NULL a failure stays
 *              recorded until a later call passes status_out.
 *   limit      sdk_decode_workspace_bytes(B, Hq, head_dim, n_atoms,
 *              max_len) <= SDK_DECODE_STATIC_WS_BYTES, else SDK_ERR_CAPACITY
 *              before anything is launched (for example one sequence with
 *              32 query heads over 32768-atom dictionaries fits up to
 *              about 8,100 tokens).
 *   zeroing    the array's header words must start at zero: they are zero
 *              when the module loads and status_out re-zeroes them; the
 *              kernels write every other byte before reading it.
 *   setup      the first call in a device's context looks up the array's
 *              address (cudaGetSymbolAddress, which may load the module);
 *              make that first call before any stream capture.  The
 *              address is kept per context and looked up again when the
 *              current context changes (after cudaDeviceReset, for one).
 *   races      there is one array per device: calls that overlap in time
 *              on a device (other streams, other host threads) race on it
 *              and give undefined results; serialise them on one stream.
 */
#define SDK_DECODE_STATIC_WS_BYTES (16u << 20)
SDK_API sdk_status sdk_decode_attn_static(const float* q, int32_t B, int32_t Hq,
                           int32_t Hkv, int32_t head_dim,
                           const void* dict_k, const void* dict_v,
                           int32_t n_atoms, const uint32_t* k_lo,
                           const uint32_t* k_full, const uint32_t* v_full,
                           int64_t cap, const int32_t* lens_host,
                           int32_t klow, int32_t khigh, int32_t top_num,
                           int32_t top_den, int32_t flags, float scale,
                           float* out, uint32_t* status_out,
                           sdk_stream_t stream);

/* Byte offsets of the decode workspace regions, for inspection by tests
 * and tools after a call (contents are valid until the next call using the
 * same workspace).  R = B*Hq query heads, L = `row` (max_len rounded up to
 * a multiple of 4). */
typedef struct {
  size_t header;     /* 256-byte status header                            */
  size_t qd;         /* float  [R][n_atoms]   QD = D_K q                  */
  size_t keys;       /* uint32 [R][L]  order-preserving keys of s_lo      */
  size_t hist1;      /* uint32 [R][4096] histogram of key bits 31..20     */
  size_t hist2;      /* uint32 [R][4096] bits 19..8 inside the bucket     */
  size_t state;      /* sdk_select_state [R]                              */
  size_t list;       /* int32  [R][L]  the selected tokens at the front
                        (unordered); with SDK_DECODE_FULL_SOFTMAX the other tokens
                        fill the back                                     */
  size_t cand_t;     /* int32  [R][L]  tokens inside the pass-1 bucket    */
  size_t cand_key;   /* uint32 [R][L]  their keys                         */
  size_t sel_score;  /* float  [R][L]  s_t of list[r][i], i < k           */
  size_t w;          /* bf16   [3][R][n_atoms] the per-atom weights w[r]
                        (softmax-normalised) as three parts, w = w[0] +
                        w[1] + w[2], each the bf16 rounding of what the
                        previous parts leave                              */
  size_t part;       /* (empty)                                           */
  size_t total;      /* total bytes                                       */
  size_t row;        /* elements per head in keys, list, cand_t, cand_key
                        and sel_score: max_len rounded up to a multiple of
                        4 (16-byte aligned rows)                          */
} sdk_decode_layout;

/* Per-head selection state in the decode workspace (region `state`).
 * Keys map a float score s to a uint32 whose unsigned order is the order
 * of s (+0 and -0 map to the same key). */
typedef struct {
  uint32_t kth_key;    /* key of the k-th largest s_lo                     */
  uint32_t k;          /* selected-set size                                */
  uint32_t n_above;    /* tokens above the pass-1 bucket                   */
  uint32_t n_cand;     /* tokens inside the pass-1 bucket                  */
  uint32_t n_sel;      /* entries written at the front of `list`           */
  uint32_t n_comp;     /* entries written at the back of `list`            */
  uint32_t eq_total;   /* tokens with key == kth_key                       */
  uint32_t eq_taken;   /* how many of those are in the selected set        */
  uint32_t max_score;  /* key of max s_t over the selected set             */
  uint32_t max_comp;   /* key of the largest s_lo outside it (0 = none)    */
  float z;             /* softmax denominator (integer softmax: E, rounded) */
  uint32_t isoft_sum[2];  /* integer softmax: E = sum of the integer
                             exponentials, low and high words              */
  uint32_t isoft_shift;   /* integer softmax: the overflow guard's shift   */
  uint32_t bracket_lo;    /* sampled bracket of the k-th key: tokens with  */
  uint32_t bracket_hi;    /*   key > hi are selected during the Klow scan,
                             lo <= key <= hi become candidates (0 and 0
                             when the selection ran by radix histograms)   */
  uint32_t select_path;   /* 0: histogram passes; 1: sampled bracket; 2:
                             bracket missed, exact re-scan of the head     */
  uint32_t pad[3];
} sdk_select_state;

SDK_API sdk_status sdk_decode_layout_of(int32_t B, int32_t Hq, int32_t head_dim,
                                int32_t n_atoms, int64_t max_len,
                                sdk_decode_layout* layout_out /* host */);

/* ------------------------------------------------------------ workspaces
 * Every workspace starts with a 256-byte header:
 *   uint32 [0] status recorded on the device (0 = none; sticky)
 *   uint32 [1] detail of the first recorded failure (e.g. the bad index)
 *   uint32 [2] encode: rows that needed the exact fallback scan
 *   uint32 [3] encode: candidate atoms re-scored in fp32
 * sdk_workspace_init zeroes the header (stream-ordered); call it once per
 * new workspace.  sdk_check_status synchronises `stream`, returns the
 * recorded status (SDK_OK if none) and clears it; `counters_out` (host,
 * nullable) receives words [0..3] before the clear.
 */
SDK_API sdk_status sdk_workspace_init(void* workspace, size_t ws_bytes,
                              sdk_stream_t stream);
SDK_API sdk_status sdk_check_status(void* workspace, sdk_stream_t stream,
                            uint32_t* counters_out);

/* Kernel timing, for measurement.  While enabled (a process-wide switch),
 * every launch of the decode attention kernel (the Khigh rescore, softmax
 * and value scatter: one per sdk_decode_attn call, one in each of stages 5
 * and 6 of sdk_decode_attn_shard) and of the tensor-core encoder (one per
 * sdk_encode / sdk_append call that takes it) is bracketed by a pair of CUDA events
 * recorded on the call's stream; the pairs are the current device's slots
 * 0, 1, 2, ... of SDK_TIMING_SLOTS, reused round-robin.  Calls captured in
 * a CUDA graph keep their slots, and every replay records them again.
 * sdk_timing_enable(on): sets the switch; turning it on (outside any stream
 * capture: it creates the current device's events the first time) restarts
 * at slot 0.
 * sdk_timing_read: waits for the events of slots 0 .. n-1, n = min(max_n,
 * slots used since the last enable, SDK_TIMING_SLOTS), writes their
 * durations in milliseconds to ms_out (host, >= max_n floats) and returns
 * n; -1 on a CUDA error (SDK_ERR_CUDA semantics).
 */
#define SDK_TIMING_SLOTS 256
SDK_API sdk_status sdk_timing_enable(int32_t on);
SDK_API int32_t sdk_timing_read(float* ms_out, int32_t max_n);

#ifdef __cplusplus
}
#endif

#endif /* SDK_H */
