// Greedy pursuit for a handful of vectors (the per-token append of decode):
// the atoms, not the vectors, are spread over the GPU, and the correlations
// come from the tensor cores.
//
// Method ("LLM Inference in a Flash!", evolve.pub review, Summary): K picks per
// vector, each the atom maximising |<r, d_i>| (ties: lowest index), coef =
// <r, d_i>, r -= coef d_i.  The review's FAQ has the codes appended at every
// generated token, i.e. a few vectors per call (one per KV head and
// sequence, for K and for V).  A vector-parallel encoder would run such a
// call on one SM.  Here CTA g owns atoms [256 g, 256 g + 256) of every
// stream's dictionary, loaded once by TMA into shared memory in the
// tcgen05 operand layout, and keeps a copy of all residuals (<= 64 rows,
// fp32).  One greedy step:
//   1. each residual row r is scaled by a power of two s (max |r s| in
//      [1, 2)), rounded to bf16 and written as the B operand;
//   2. tcgen05.mma (M = 128 atoms, N = rows, K = 16, fp32 accumulation in
//      tensor memory) gives c~ ~ s <r, d> for every (atom, row) of the slice;
//   3. per warp (32 atoms) and row, every atom with |c~| >= max |c~| - band
//      is re-scored with the CUDA-core encoder's exact arithmetic (an fp32
//      FMA chain over k = 0..D-1 on the unscaled residual).  band =
//      2^-7 ||r s|| max||d|| is twice a bound on |c~ - s c_chain| (bf16
//      rounding of r s: 2^-9; tensor-core accumulation of D exact products:
//      < 2^-16; the chain's own rounding: < 2^-16; relative to
//      ||r s|| ||d||), so the warp's exact argmax is always re-scored;
//   4. the slice winner (|c|, index, sign, step tag) is published as one
//      64-bit word; every CTA reads all CTAs' words for every row, polling
//      until each carries this step's tag (no separate grid barrier), and
//      takes the same maximum, so all CTAs hold the same pick;
//   5. r = fmaf(-coef, d, r) in fp32 (d read from the dictionary in L2);
//      CTA 0 writes the code words.
// Picks, coefficients and residuals are therefore bit-identical to the
// CUDA-core encoder's.  Up to two streams share one launch (the K and V
// vectors of an append, each with its own dictionary and the same number
// of rows <= 32): stream s owns rows 32 s .. 32 s + m - 1.  In append mode
// CTA 0 writes the words straight into the code store (full words and, for
// keys, the first-3 planes).
// The launch is cooperative, so every CTA is resident while the others
// poll for its words.  Every wait (TMA, MMA, word polls) is bounded by 1 s
// of %globaltimer; on expiry the CTA records SDK_ERR_TIMEOUT and leaves the
// loop, and the CTAs polling for its words then time out in turn.
#include <stdlib.h>
#include <string.h>

#include "tc_ptx.cuh"

namespace sdk {

namespace {

using namespace tc;

constexpr int kThreads = 256;
constexpr int kSlots = 64;          // residual rows per call
constexpr int kTileAtoms = 128;     // MMA M
constexpr int kMaxTiles = 2;        // atoms per CTA <= 256
constexpr int kMaxGrid = 1024;
constexpr int kWarpCand = 512;      // re-score list of a warp: 16 rows x 32 atoms
constexpr int kBatch = 16;          // 16-byte word loads in flight per thread

template <int D>
struct SCfg {
  static constexpr int KB = D / 64;                      // 128-byte K blocks
  static constexpr int KSTEPS = D / 16;
  static constexpr int kTileBytes = kTileAtoms * D * 2;  // one 128-atom tile
  static constexpr int kOffB = 2 * kMaxTiles * kTileBytes;
  static constexpr int kBBytes = kSlots * D * 2;         // 64 bf16 rows per stream
  static constexpr int kOffR = kOffB + 2 * kBBytes;
  static constexpr int kRStride = D + 4;                 // floats per residual row (padded)
  static constexpr int kOffCand = kOffR + kSlots * kRStride * 4;
  static constexpr int kOffMisc = kOffCand + 8 * kWarpCand * 4;
  static constexpr int kMiscBytes = 4096;
  static constexpr int kSmem = kOffMisc + kMiscBytes + 1024;   // + alignment slack
  static_assert(kSmem <= 232448, "exceeds the 227 KB shared memory of one sm_100 CTA");
};

struct SmallParams {
  const void* x[2];
  const uint16_t* dict[2];
  int m[2];              // rows per stream (dual: equal, <= 32)
  int streams;
  int x_dtype;
  int n;                 // atoms per dictionary
  int k_atoms;
  int slice;             // atoms per CTA, multiple of 32, <= 256
  // outputs: plain mode writes codes[s][i * k_atoms + j]; append mode writes
  // codes[s][(bk * cap + t) * rs + j] (and lo[s][(bk * 3 + j) * cap + t] for
  // j < 3 when lo[s] is set) with bk = i / n_new, t = lens[bk / Hkv] + i % n_new
  uint32_t* codes[2];
  float* rsq[2];
  int append;
  uint32_t* lo[2];
  int64_t cap;
  int n_new, Hkv, rs;
  int lens[32];
  WsHeader* hdr;
  unsigned long long* words;   // [2][grid][64], zero before the launch
  unsigned long long wait_ns;  // limit of every poll for another CTA's word
};

// Word of a slice winner: bits 63..32 |c| (fp32 bits), 31..17 0x7fff - index,
// 16 sign of c, 15..1 step tag, 0 set when the slice has a winner.  The
// maximum word is the largest |c|, then the lowest index.
__device__ __forceinline__ unsigned long long win_word(float c, uint32_t idx) {
  const float a = fabsf(c);
  if (!(a >= 0.0f)) return 0ull;  // NaN never wins (as in the CUDA-core scan)
  return ((unsigned long long)__float_as_uint(a) << 32) |
         ((unsigned long long)(0x7FFFu - idx) << 17) |
         ((unsigned long long)(__float_as_uint(c) >> 31) << 16) | 1ull;
}
__device__ __forceinline__ uint32_t word_tag(unsigned long long w) {
  return (uint32_t)(w >> 1) & 0x7FFFu;
}

__device__ __forceinline__ void st_relaxed_u64(unsigned long long* p, unsigned long long v) {
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
// two adjacent words (16-byte aligned); each word is read single-copy atomic
__device__ __forceinline__ ulonglong2 ld_relaxed_v2(const unsigned long long* p) {
  ulonglong2 v;
  asm volatile("ld.relaxed.gpu.global.v2.u64 {%0, %1}, [%2];" : "=l"(v.x), "=l"(v.y) : "l"(p)
               : "memory");
  return v;
}

// Maximum over the words of one slot pair from CTAs c0, c0 + cstep, ...:
// all loads issued at once, each word polled until it carries `tag`
// (bounded by limit_ns and the CTA's abort flag).  False on timeout.
template <int B>
__device__ __forceinline__ bool gather_words(const unsigned long long* wb, int c0, int cstep, int G,
                                             int vr, bool v1, uint32_t tag,
                                             volatile uint32_t* abort_flag,
                                             unsigned long long limit_ns, unsigned long long& mx0,
                                             unsigned long long& mx1) {
  for (int cb = c0; cb < G; cb += cstep * B) {
    ulonglong2 w[B];
#pragma unroll
    for (int u = 0; u < B; ++u) {
      const int c = cb + u * cstep;
      if (c < G) w[u] = ld_relaxed_v2(wb + (size_t)c * 64 + vr);
    }
#pragma unroll
    for (int u = 0; u < B; ++u) {
      const int c = cb + u * cstep;
      if (c >= G) break;
      ulonglong2 x = w[u];
      if (word_tag(x.x) != tag || (v1 && word_tag(x.y) != tag)) {
        const uint64_t t0 = tc::globaltimer();
        while (true) {
          x = ld_relaxed_v2(wb + (size_t)c * 64 + vr);
          if (word_tag(x.x) == tag && (!v1 || word_tag(x.y) == tag)) break;
          if (*abort_flag || tc::globaltimer() - t0 > limit_ns) return false;
          __nanosleep(20);
        }
      }
      mx0 = max(mx0, x.x & ~0xFFFEull);
      if (v1) mx1 = max(mx1, x.y & ~0xFFFEull);
    }
  }
  return true;
}

// <r, d> as the CUDA-core encoder computes it: an fp32 FMA chain over
// k = 0..D-1.  d is atom ai of a 128-atom tile in the swizzled K-major
// operand layout, r a residual row in shared memory.
template <int D>
__device__ __forceinline__ float exact_chain(const uint8_t* base, int ai, const float4* rr) {
  const uint8_t* row = base + ai * 128;
  const int sw = ai & 7;
  float c = 0.0f;
#pragma unroll
  for (int kc = 0; kc < D / 8; ++kc) {
    const uint4 w = *reinterpret_cast<const uint4*>(row + (kc >> 3) * (128 * 128) +
                                                    (((kc & 7) ^ sw) << 4));
    const float4 a = rr[2 * kc], b = rr[2 * kc + 1];
    c = fmaf(a.x, bf16_lo(w.x), c);
    c = fmaf(a.y, bf16_hi(w.x), c);
    c = fmaf(a.z, bf16_lo(w.y), c);
    c = fmaf(a.w, bf16_hi(w.y), c);
    c = fmaf(b.x, bf16_lo(w.z), c);
    c = fmaf(b.y, bf16_hi(w.z), c);
    c = fmaf(b.z, bf16_lo(w.w), c);
    c = fmaf(b.w, bf16_hi(w.w), c);
  }
  return c;
}

// 2^(127 - e) for the exponent e of max |r| (clamped so the scale and the
// scaled maximum stay normal): max |r s| in [1, 2) for normal maxima.
__device__ __forceinline__ float row_scale(uint32_t maxbits) {
  int e = (int)((maxbits >> 23) & 0xFFu);
  e = e < 1 ? 1 : (e > 253 ? 253 : e);
  return __uint_as_float((uint32_t)(254 - e) << 23);
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    encode_small_kernel(const __grid_constant__ CUtensorMap map0,
                        const __grid_constant__ CUtensorMap map1, SmallParams p) {
  using C = SCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_smem_1k(smem_raw);
  float* rT = reinterpret_cast<float*>(smem + C::kOffR);           // [64][D + 4] residual rows
  uint32_t* cand = reinterpret_cast<uint32_t*>(smem + C::kOffCand);
  uint8_t* misc = smem + C::kOffMisc;
  unsigned long long* s_key = reinterpret_cast<unsigned long long*>(misc);          // 64
  unsigned long long* s_best = s_key + kSlots;                                       // 64
  uint64_t* bars = reinterpret_cast<uint64_t*>(s_best + kSlots);                     // 2
  float* s_rn = reinterpret_cast<float*>(bars + 2);                                  // 64
  uint32_t* s_rmax = reinterpret_cast<uint32_t*>(s_rn + kSlots);                     // 2 x 64
  float* s_band = reinterpret_cast<float*>(s_rmax + 2 * kSlots);                     // 64
  uint32_t* s_dmax = reinterpret_cast<uint32_t*>(s_band + kSlots);                   // 2
  volatile uint32_t* s_abort = s_dmax + 2;
  volatile uint32_t* s_tmem = s_dmax + 3;
  const uint32_t bar_load = smem_u32(&bars[0]);
  const uint32_t bar_mma = smem_u32(&bars[1]);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x, g = blockIdx.x;
  const int S = p.slice, n = p.n;
  const int a0 = g * S;
  const bool dual = p.streams == 2;
  const int ns = dual ? 2 : 1;
  // 128-atom tiles of this CTA's slice that hold atoms below n
  const int tiles = min((S + kTileAtoms - 1) / kTileAtoms, (n - a0 + kTileAtoms - 1) / kTileAtoms);
  const int nvalid = dual ? p.m[0] + p.m[1] : p.m[0];
  int lg_nv = 0;
  while ((1 << lg_nv) < nvalid) ++lg_nv;
  const int nv_pad = 1 << lg_nv;   // rows rounded up to a power of two
  auto vr_stream = [&](int vr) { return dual ? (vr >> 5) : 0; };
  auto vr_row = [&](int vr) { return dual ? (vr & 31) : vr; };
  auto vr_valid = [&](int vr) { return vr_row(vr) < p.m[vr_stream(vr)]; };
  auto tile_addr = [&](int s, int t) { return smem + (s * kMaxTiles + t) * C::kTileBytes; };

  if (tid == 0) {
    *s_abort = 0u;
    s_dmax[0] = s_dmax[1] = 0u;
    mbar_init(bar_load, 1);
    mbar_init(bar_mma, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32((const void*)s_tmem)),
                 "r"(128)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (tid < kSlots) {
    s_key[tid] = 0ull;
    s_best[tid] = 0ull;
    s_rn[tid] = 0.0f;
    s_rmax[tid] = 0u;
    s_rmax[kSlots + tid] = 0u;
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;

  // dictionary slices: TMA, 128-byte swizzle, K-major (atoms past n read 0)
  if (tid == 0) {
    mbar_expect_tx(bar_load, (uint32_t)(ns * tiles * C::kTileBytes));
    for (int s = 0; s < ns; ++s)
      for (int t = 0; t < tiles; ++t)
#pragma unroll
        for (int kb = 0; kb < C::KB; ++kb)
          tma_load_2d(smem_u32(tile_addr(s, t)) + kb * (kTileAtoms * 128), s == 0 ? &map0 : &map1,
                      kb * 64, a0 + t * kTileAtoms, bar_load);
  }
  // residuals <- x; B operands zeroed (rows past m stay zero)
  for (int e = tid; e < D * kSlots; e += kThreads) {
    const int vr = e / D, k = e % D;
    float xv = 0.0f;
    if (vr_valid(vr)) {
      const int s = vr_stream(vr);
      const int64_t o = (int64_t)vr_row(vr) * D + k;
      xv = p.x_dtype == SDK_F32 ? reinterpret_cast<const float*>(p.x[s])[o]
                                : bf16_lo(reinterpret_cast<const uint16_t*>(p.x[s])[o]);
      atomicMax(&s_rmax[vr], __float_as_uint(fabsf(xv)));
    }
    rT[vr * C::kRStride + k] = xv;
  }
  for (int e = tid; e < 2 * C::kBBytes / 16; e += kThreads)
    reinterpret_cast<uint4*>(smem + C::kOffB)[e] = make_uint4(0u, 0u, 0u, 0u);
  {
    uint32_t dummy = 0u;
    if (!mbar_wait(bar_load, 0u, &dummy)) {
      record_error(p.hdr, SDK_ERR_TIMEOUT, 0x61000000u | (uint32_t)g);
      *s_abort = 1u;
    }
  }
  __syncthreads();
  // max ||d|| over the slice, per stream
  if (!*s_abort)
    for (int s = 0; s < ns; ++s) {
      const int al = tid;
      if (al < S && a0 + al < n) {
        const int t = al / kTileAtoms, ai = al % kTileAtoms;
        const uint8_t* base = tile_addr(s, t);
        float sq = 0.0f;
#pragma unroll
        for (int kc = 0; kc < D / 8; ++kc) {
          const uint4 w = *reinterpret_cast<const uint4*>(
              base + (kc >> 3) * (kTileAtoms * 128) + ai * 128 + (((kc & 7) ^ (ai & 7)) << 4));
          const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            const float lo = bf16_lo(wv[h]), hi = bf16_hi(wv[h]);
            sq = fmaf(lo, lo, sq);
            sq = fmaf(hi, hi, sq);
          }
        }
        atomicMax(&s_dmax[s], __float_as_uint(sqrtf(sq)));
      }
    }
  __syncthreads();

  // MMA shape per stream: N = rows rounded up to 16; accumulator of tile t
  // at TMEM columns t*64 (+ 32 for stream 1)
  const int N0 = (p.m[0] + 15) & ~15;
  const int N1 = dual ? (p.m[1] + 15) & ~15 : 0;
  const int q = warp & 3, tw = warp >> 2;
  const int a_loc = tw * kTileAtoms + q * 32 + lane;
  const bool atom_ok = tw < tiles && a_loc < S && a0 + a_loc < n;

  // valid rows in slot order: vi -> slot (stream 1 starts at slot 32)
  auto slot_of = [&](int vi) { return dual && vi >= p.m[0] ? 32 + (vi - p.m[0]) : vi; };
  // 16-column groups of the accumulator that hold valid rows
  auto group_valid = [&](int cg) {
    return dual ? 16 * (cg & 1) < p.m[cg >> 1] : 16 * cg < p.m[0];
  };
  // exact correlation of residual row vr with slice atom al: the CUDA-core
  // encoder's fp32 FMA chain over k = 0..D-1
  auto chain = [&](int vr, int al) -> float {
    return exact_chain<D>(tile_addr(vr_stream(vr), al / kTileAtoms), al % kTileAtoms,
                          reinterpret_cast<const float4*>(rT + vr * C::kRStride));
  };
  // word pairs (two adjacent slots) per CTA that hold valid rows
  const int np0 = (p.m[0] + 1) >> 1, np1 = dual ? (p.m[1] + 1) >> 1 : 0;
  const int npairs = np0 + np1;
  int lg_np = 0;
  while ((1 << lg_np) < npairs) ++lg_np;
  const int np_pad = 1 << lg_np;   // <= 32
  const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16) + tw * 64;

  // bf16(r s) of 8 residual components into row vr's B operand; returns
  // their sum of squares
  auto put_b = [&](int vr, int c, const float4& x0, const float4& x1, float sc) -> float {
    const float v[8] = {x0.x * sc, x0.y * sc, x0.z * sc, x0.w * sc,
                        x1.x * sc, x1.y * sc, x1.z * sc, x1.w * sc};
    uint32_t w[4];
    float sq = 0.0f;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * u], v[2 * u + 1]);
      w[u] = *reinterpret_cast<const uint32_t*>(&h);
      sq = fmaf(v[2 * u], v[2 * u], sq);
      sq = fmaf(v[2 * u + 1], v[2 * u + 1], sq);
    }
    const int s = vr_stream(vr), row = vr_row(vr);
    const int kb = c >> 3, c16 = c & 7;
    *reinterpret_cast<uint4*>(smem + C::kOffB + s * C::kBBytes + kb * (kSlots * 128) + row * 128 +
                              ((c16 ^ (row & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
    return sq;
  };
  // step 0's B operand: r = x, scale from max |x|
  for (int e = tid; e < (D / 8) << lg_nv; e += kThreads) {
    const int vi = e & (nv_pad - 1), c = e >> lg_nv;
    if (vi >= nvalid) continue;
    const int vr = slot_of(vi);
    const float4* r4 = reinterpret_cast<const float4*>(rT + vr * C::kRStride + 8 * c);
    atomicAdd(&s_rn[vr], put_b(vr, c, r4[0], r4[1], row_scale(s_rmax[vr])));
  }
  fence_proxy_async();
  __syncthreads();

  // Per step j: s_rmax[j & 1] = max |r_j| (r_j's zero test; the scale of
  // r_{j+1}'s operand), s_rn = ||r_j s||^2 of the operand in B.
  for (int j = 0; j < p.k_atoms && !*s_abort; ++j) {
    const int buf = j & 1;
    const uint32_t tag = (uint32_t)(j + 1);
    const uint32_t* rmax = s_rmax + buf * kSlots;
    uint32_t* rmax_next = s_rmax + (buf ^ 1) * kSlots;
    // 1. correlations of the slice with all rows; meanwhile each row's band
    if (tid == 0) {
      tc_fence_after();
      for (int s = 0; s < ns; ++s) {
        const int N = s == 0 ? N0 : N1;
        const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) |
                               ((uint32_t)(kTileAtoms >> 4) << 24);
        const uint64_t bdesc = smem_desc(smem_u32(smem + C::kOffB + s * C::kBBytes));
        for (int t = 0; t < tiles; ++t) {
          const uint64_t adesc = smem_desc(smem_u32(tile_addr(s, t)));
#pragma unroll
          for (int ks = 0; ks < C::KSTEPS; ++ks) {
            // descriptor start addresses advance in 16-byte units
            const uint32_t aoff = (ks >> 2) * (kTileAtoms * 128) + (ks & 3) * 32;
            const uint32_t boff = (ks >> 2) * (kSlots * 128) + (ks & 3) * 32;
            tc_mma(tmem + t * 64 + s * 32, adesc + (aoff >> 4), bdesc + (boff >> 4), idesc,
                   ks > 0 ? 1u : 0u);
          }
        }
      }
      tc_commit(bar_mma);
    }
    if (tid < kSlots && vr_valid(tid))
      s_band[tid] = 0.0078125f * sqrtf(s_rn[tid]) * __uint_as_float(s_dmax[vr_stream(tid)]) * 1.01f +
                    7.7e-34f;
    if (tid == 0 && !mbar_wait(bar_mma, (uint32_t)(j & 1), s_abort)) {
      record_error(p.hdr, SDK_ERR_TIMEOUT, 0x62000000u | (uint32_t)g);
      *s_abort = 1u;
    }
    __syncthreads();
    if (*s_abort) break;
    tc_fence_after();
    // state for the exchange and the fused update of this step
    if (tid < kSlots) {
      s_best[tid] = 0ull;
      s_rn[tid] = 0.0f;
      rmax_next[tid] = 0u;
    }
    // 2. per warp (32 atoms, one per lane) and row: the largest |c~|, every
    // atom not provably below it (|c~| >= max - band) into the warp's list,
    // then the list re-scored exactly, one entry per lane.  Rows are taken 16
    // accumulator columns at a time.
    if (tw < tiles) {
      uint32_t* wl = cand + warp * kWarpCand;
      int cnt = 0;
      // re-score the listed candidates, one entry per lane
      auto flush = [&]() {
        __syncwarp();
        for (int i = lane; i < cnt; i += 32) {
          const uint32_t cw = wl[i];
          const int vr = (int)(cw >> 16), al = (int)(cw & 0xFFFFu);
          const unsigned long long key = win_word(chain(vr, al), (uint32_t)(a0 + al));
          if (key) atomicMax(&s_key[vr], key);
        }
        __syncwarp();
        cnt = 0;
      };
      for (int cg = 0; cg < 4; ++cg) {
        if (!group_valid(cg)) continue;
        uint32_t v[16];
        tmem_ld16(taddr + cg * 16, v);
        tmem_ld_wait();
        // rows of the group to scan (valid and not zero) and their bands,
        // lane u holding row u's
        const int vr_l = cg * 16 + (lane & 15);
        const bool row_l = vr_valid(vr_l) && rmax[vr_l] != 0u;
        const float band_l = s_band[vr_l];
        const uint32_t rows = __ballot_sync(0xffffffffu, row_l) & 0xFFFFu;
        uint32_t bal[16];
        int gcnt = 0;
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          const bool row = (rows >> u) & 1u;
          const float a = fabsf(__uint_as_float(v[u]));
          const uint32_t b = (row && atom_ok && a == a) ? __float_as_uint(a) : 0u;
          const float wmax = __uint_as_float(__reduce_max_sync(0xffffffffu, b));
          const float band = __shfl_sync(0xffffffffu, band_l, u);
          bal[u] = __ballot_sync(0xffffffffu, row && atom_ok && !(a < wmax - band));
          gcnt += __popc(bal[u]);
        }
        // the candidates of all groups go through one round of re-scoring,
        // unless the list would overflow first
        if (cnt + gcnt > kWarpCand) flush();
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          if ((bal[u] >> lane) & 1u)
            wl[cnt + __popc(bal[u] & ((1u << lane) - 1u))] =
                ((uint32_t)(cg * 16 + u) << 16) | (uint32_t)a_loc;
          cnt += __popc(bal[u]);
        }
      }
      flush();
    }
    tc_fence_before();
    // a zero row: every chain gives +0, the slice's first atom wins
    if (tid < kSlots && vr_valid(tid) && rmax[tid] == 0u)
      atomicMax(&s_key[tid], win_word(0.0f, (uint32_t)a0));
    __syncthreads();
    // 3. publish the slice winners, then take the maximum over all slices:
    // 16-byte loads of two adjacent slots' words, polled until every valid
    // one carries this step's tag
    unsigned long long* wb = p.words + (size_t)buf * G * kSlots;
    if (tid < kSlots && vr_valid(tid))
      st_relaxed_u64(wb + (size_t)g * kSlots + tid, s_key[tid] | ((unsigned long long)tag << 1));
    {
      // thread -> one word pair (tid mod np_pad) and every (256 / np_pad)-th
      // CTA; all of its loads in flight at once
      bool ok = true;
      const int pr = tid & (np_pad - 1);
      if (pr < npairs) {
        const int vr = pr < np0 ? 2 * pr : 32 + 2 * (pr - np0);
        const bool v1 = vr_valid(vr + 1);
        const int cstep = kThreads >> lg_np;
        const int c0 = tid >> lg_np;
        unsigned long long mx0 = 0ull, mx1 = 0ull;
        if (cstep * 4 >= G)
          ok = gather_words<4>(wb, c0, cstep, G, vr, v1, tag, s_abort, p.wait_ns, mx0, mx1);
        else
          ok = gather_words<kBatch>(wb, c0, cstep, G, vr, v1, tag, s_abort, p.wait_ns, mx0,
                                    mx1);
        if (mx0) atomicMax(&s_best[vr], mx0);
        if (mx1) atomicMax(&s_best[vr + 1], mx1);
      }
      if (!ok) {
        if (!*s_abort) record_error(p.hdr, SDK_ERR_TIMEOUT, 0x63000000u | (uint32_t)g);
        *s_abort = 1u;
      }
    }
    __syncthreads();
    if (*s_abort) break;
    // 4. pick and coefficient of every row (read by every thread of the row
    // from the maximum word), r_{j+1} = fmaf(-coef, d, r_j) in fp32 (the
    // same in every CTA), and r_{j+1}'s operand scaled as r_j's maximum
    // asks (|r_{j+1} s| <= ||r_j s|| <= 2 sqrt(D): no overflow)
    if (tid < kSlots) s_key[tid] = 0ull;
    for (int e = tid; e < (D / 8) << lg_nv; e += kThreads) {
      const int vi = e & (nv_pad - 1), c = e >> lg_nv;
      if (vi >= nvalid) continue;
      const int vr = slot_of(vi);
      const int s = vr_stream(vr);
      const unsigned long long bw = s_best[vr];
      int pick = 0;
      float cf = 0.0f;   // every |c| NaN: atom 0 with coefficient 0, as the CUDA-core scan
      if (bw & 1ull) {
        pick = (int)(0x7FFFu - (uint32_t)((bw >> 17) & 0x7FFFu));
        const float a = __uint_as_float((uint32_t)(bw >> 32));
        cf = ((bw >> 16) & 1ull) ? -a : a;
      }
      const uint4 w = __ldg(reinterpret_cast<const uint4*>(p.dict[s] + (int64_t)pick * D) + c);
      float4* r4 = reinterpret_cast<float4*>(rT + vr * C::kRStride + 8 * c);
      float4 x0 = r4[0], x1 = r4[1];
      x0.x = fmaf(-cf, bf16_lo(w.x), x0.x);
      x0.y = fmaf(-cf, bf16_hi(w.x), x0.y);
      x0.z = fmaf(-cf, bf16_lo(w.y), x0.z);
      x0.w = fmaf(-cf, bf16_hi(w.y), x0.w);
      x1.x = fmaf(-cf, bf16_lo(w.z), x1.x);
      x1.y = fmaf(-cf, bf16_hi(w.z), x1.y);
      x1.z = fmaf(-cf, bf16_lo(w.w), x1.z);
      x1.w = fmaf(-cf, bf16_hi(w.w), x1.w);
      r4[0] = x0;
      r4[1] = x1;
      const float m8 = fmaxf(fmaxf(fmaxf(fabsf(x0.x), fabsf(x0.y)), fmaxf(fabsf(x0.z), fabsf(x0.w))),
                             fmaxf(fmaxf(fabsf(x1.x), fabsf(x1.y)), fmaxf(fabsf(x1.z), fabsf(x1.w))));
      // NaN components: the row is degenerate; the rest sets the scale
      if (m8 > 0.0f) atomicMax(&rmax_next[vr], __float_as_uint(m8));
      atomicAdd(&s_rn[vr], put_b(vr, c, x0, x1, row_scale(rmax[vr])));
      if (c == 0 && g == 0) {
        const int i = vr_row(vr);
        const uint32_t word = make_word(cf, (uint32_t)pick);
        if (!p.append) {
          p.codes[s][(int64_t)i * p.k_atoms + j] = word;
        } else {
          const int bk = i / p.n_new;
          const int64_t t = (int64_t)p.lens[bk / p.Hkv] + i % p.n_new;
          p.codes[s][((int64_t)bk * p.cap + t) * p.rs + j] = word;
          if (p.lo[s] != nullptr && j < kLoPlanes)
            p.lo[s][((int64_t)bk * kLoPlanes + j) * p.cap + t] = word;
        }
      }
    }
    fence_proxy_async();
    __syncthreads();
  }
  if (g == 0 && !*s_abort && tid < kSlots && vr_valid(tid)) {
    const int s = vr_stream(tid);
    if (p.rsq[s] != nullptr) {
      float sq = 0.0f;
      for (int k = 0; k < D; ++k) {
        const float r = rT[tid * C::kRStride + k];
        sq = fmaf(r, r, sq);
      }
      p.rsq[s][vr_row(tid)] = sq;
    }
  }
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(128)
                 : "memory");
  }
}

bool small_enabled() {
  static int on = -1;
  if (on < 0) {
    const char* v = getenv("SDK_ENCODE_SMALL");
    on = (v != nullptr && v[0] == '0') ? 0 : 1;
  }
  return on == 1;
}

bool make_map(CUtensorMap* map, const uint16_t* dict, int D, int n) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)n};
  const cuuint64_t strides[1] = {(cuuint64_t)D * 2};
  const cuuint32_t box[2] = {64u, (cuuint32_t)kTileAtoms};
  const cuuint32_t estr[2] = {1u, 1u};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(dict), dims, strides,
            box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

size_t encode_small_scratch_bytes() { return (size_t)2 * kMaxGrid * kSlots * 8; }

sdk_status launch_encode_small(const SmallEncode& e, void* scratch, size_t scratch_bytes,
                               cudaStream_t stream, bool* taken) {
  *taken = false;
  if (!small_enabled()) return SDK_OK;
  const int D = e.head_dim;
  if (D != 64 && D != 128) return SDK_OK;
  if (e.streams < 1 || e.streams > 2) return SDK_OK;
  const int64_t m0 = e.p[0].n_vec, m1 = e.streams == 2 ? e.p[1].n_vec : 0;
  if (e.streams == 1 && (m0 < 1 || m0 > kSlots)) return SDK_OK;
  if (e.streams == 2 && (m0 < 1 || m0 > kSlots / 2 || m1 != m0)) return SDK_OK;
  if (e.streams == 2 && (e.p[0].n != e.p[1].n || e.p[0].k_atoms != e.p[1].k_atoms)) return SDK_OK;
  if (e.p[0].k_atoms > 0x7FFF) return SDK_OK;
  if (e.append && (e.B > 32 || e.p[0].k_atoms != kAtoms || e.n_new < 1)) return SDK_OK;
  if (scratch_bytes < encode_small_scratch_bytes()) return SDK_OK;
  const int n = e.p[0].n;
  int dev = 0, coop = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SDK_ERR_CUDA;
  if (cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev) != cudaSuccess || !coop)
    return SDK_OK;
  const int sms = num_sms();
  // 256 atoms (two 128-atom tiles) per CTA: the fewest CTAs, so the fewest
  // words to exchange per step
  const int slice = kMaxTiles * kTileAtoms;
  const int grid = (n + slice - 1) / slice;
  if (grid > sms) return SDK_OK;
  if (grid > kMaxGrid) return SDK_OK;
  CUtensorMap maps[2];
  for (int s = 0; s < e.streams; ++s)
    if (!make_map(&maps[s], e.p[s].dict, D, n)) return SDK_OK;
  if (e.streams == 1) maps[1] = maps[0];
  const void* fn = D == 128 ? (const void*)encode_small_kernel<128> : (const void*)encode_small_kernel<64>;
  const int smem = D == 128 ? SCfg<128>::kSmem : SCfg<64>::kSmem;
  static unsigned long long attr_set = 0ull;
  if (device_needs_setup(&attr_set)) {
    cudaFuncSetAttribute(encode_small_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         SCfg<128>::kSmem);
    cudaFuncSetAttribute(encode_small_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         SCfg<64>::kSmem);
    device_setup_done(&attr_set);
  }
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, kThreads, smem) != cudaSuccess)
    return SDK_ERR_CUDA;
  if ((int64_t)per_sm * sms < grid) return SDK_OK;  // not every CTA could be resident

  SmallParams sp;
  memset(&sp, 0, sizeof(sp));
  for (int s = 0; s < 2; ++s) {
    const bool used = s < e.streams;
    const EncodeParams& ps = e.p[used ? s : 0];
    sp.x[s] = ps.x;
    sp.dict[s] = ps.dict;
    sp.codes[s] = ps.codes;
    sp.rsq[s] = used ? ps.rsq : nullptr;
    sp.lo[s] = used ? e.lo[s] : nullptr;
    sp.m[s] = used ? (int)ps.n_vec : 0;
  }
  sp.streams = e.streams;
  sp.x_dtype = e.p[0].x_dtype;
  sp.n = n;
  sp.k_atoms = e.p[0].k_atoms;
  sp.slice = slice;
  sp.append = e.append ? 1 : 0;
  sp.cap = e.cap;
  sp.n_new = e.n_new;
  sp.Hkv = e.Hkv;
  sp.rs = e.append ? e.rs : kAtoms;
  for (int b = 0; e.append && b < e.B; ++b) sp.lens[b] = e.lens[b];
  sp.hdr = e.p[0].hdr;
  sp.words = reinterpret_cast<unsigned long long*>(scratch);
  sp.wait_ns = exchange_wait_ns();
  if (cudaMemsetAsync(sp.words, 0, (size_t)2 * grid * kSlots * 8, stream) != cudaSuccess)
    return SDK_ERR_CUDA;
  *taken = true;
  void* args[] = {&maps[0], &maps[1], &sp};
  const cudaError_t err =
      cudaLaunchCooperativeKernel(fn, dim3((unsigned)grid), dim3(kThreads), args, (size_t)smem, stream);
  return err == cudaSuccess ? SDK_OK : SDK_ERR_CUDA;
}

}  // namespace sdk
