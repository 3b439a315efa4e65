// Greedy pursuit encoder on the 5th-generation tensor cores (sm_100a).
//
// Method ("LLM Inference in a Flash!", evolve.pub review, Summary): every
// vector x gets K picks; a pick is i* = argmax_i |<r, d_i>| over the whole
// dictionary, coef = <r, d_i*>, r -= coef * d_i* (projection-based greedy
// pursuit, no least-squares refit).
//
// Design (one persistent CTA per SM, 18 warps, warp-specialised):
//   warp 0      TMA producer: streams the operand copy of the dictionary
//               through a 4-stage shared-memory ring in 128-atom tiles
//               (128B-swizzled, K-major), the same dictionary 16 times per
//               row tile.
//   warp 1      MMA issuer: allocates 512 TMEM columns; for every atom tile
//               issues tcgen05.mma kind::f16 (M=128, N=128, K=16, fp32
//               accumulate) for two 128-row sets of residuals (A operand in
//               shared memory) into one of two TMEM accumulator buffers;
//               tcgen05.commit frees the ring stage and hands the buffer to
//               the epilogue.
//   warps 2..17 epilogue: two threads per residual row (64 columns each of
//               every 128-atom tile).  tcgen05.ld brings a thread's
//               correlations to registers, the buffer is released at once,
//               and the thread keeps the running maximum
//               B of |c~| plus every atom with |c~| >= B - band.  band is
//               twice a rigorous bound on the error of c~ (operand rounding
//               of r and of the dictionary by Cauchy-Schwarz, plus
//               accumulation slack), so the exact fp32 argmax is always
//               among the kept candidates.  After the last atom tile of a
//               step the candidates are re-scored in fp32 (k = 0..D-1 FMA
//               order over the bf16 atoms, the same arithmetic as the
//               CUDA-core encoder), the row's lead thread writes the pick,
//               r is updated in fp32 (global scratch, L2-resident) and its
//               rounded copy becomes the next step's A operand.  A row whose
//               candidate list overflows is re-picked by an exact fp32 scan
//               of all atoms shared by its warp (counted in the workspace
//               header).
// Operands: fp16 by default.  The bf16 atoms are copied once per call as
// fp16(t d) with a power-of-two t (exact for every entry within 29 binades
// of the largest), and each A row holds fp16(s r) with a per-row power of
// two s, so |c~ - s t c| is about 8x tighter than with bf16 operands at the
// same MMA rate; fewer atoms fall inside the band.  Setting the environment
// variable SDK_ENCODE_OPERANDS=bf16 selects bf16 operands (the atoms as
// given, t = 1; the row scale s is kept).  Either way the picks are the
// exact fp32 argmax.
// Every wait on an mbarrier is bounded (1 s of %globaltimer); on expiry the
// CTA records SDK_ERR_TIMEOUT, stops issuing work, lets in-flight copies and
// MMAs finish (bounded), frees its TMEM and exits.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <stdlib.h>
#include <string.h>

#include "tc_ptx.cuh"

namespace sdk {
namespace tc {

constexpr int kRows = 128;                 // rows per set (TMEM lanes, MMA M)
constexpr int kSets = 2;                   // row sets per CTA
constexpr int kTileRows = kRows * kSets;   // vectors per row tile
constexpr int kAtomTile = 128;             // atoms per B tile (MMA N)
constexpr int kStages = 4;
constexpr int kCand = 8;                   // candidates kept per thread
constexpr int kEpiWarps = 16;
constexpr int kEpiThreads = 32 * kEpiWarps;
constexpr int kLeadWarps = kEpiWarps / 2;  // warps owning whole rows
constexpr int kThreads = 32 * (2 + kEpiWarps);
constexpr int kMaxCtas = 160;
constexpr int kTmemCols = 512;

template <int D>
struct Cfg {
  static constexpr int KB = D / 64;                   // 128-byte K blocks
  static constexpr int KSTEPS = D / 16;               // MMAs per row set
  static constexpr int kStageBytes = kAtomTile * D * 2;
  static constexpr int kABytes = kRows * D * 2;       // one row set
  static constexpr int kOffA = kStages * kStageBytes;
  static constexpr int kOffCw = kOffA + kSets * kABytes;          // candidate words
  static constexpr int kOffBest = kOffCw + kEpiThreads * kCand * 4;
  static constexpr int kOffCnt = kOffBest + kEpiThreads * 4;
  static constexpr int kOffBand = kOffCnt + kEpiThreads * 4;
  static constexpr int kOffAct = kOffBand + kTileRows * 4;
  static constexpr int kOffScl = kOffAct + kTileRows * 4;          // per-row A scale
  static constexpr int kOffFr = kOffScl + kTileRows * 4;          // fallback residuals
  // push staging (tile loop) shares the fallback scratch (step end only)
  static constexpr int kOffStg = kOffFr;
  static_assert(kEpiWarps * 32 <= kLeadWarps * D, "staging must fit the fallback scratch");
  static constexpr int kOffRes = kOffFr + kLeadWarps * D * 4;      // per-thread picks
  static constexpr int kOffBar = kOffRes + kEpiThreads * 12;
  static constexpr int kNumBars = 2 * kStages + 2 + 2 + 1 + 1;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  // + alignment slack; at least 116 KB so that one CTA (which holds all 512
  // TMEM columns) is resident per SM
  static constexpr int kSmemUsed = kOffMisc + 64 + 1024;
  static constexpr int kSmem = kSmemUsed > 116 * 1024 ? kSmemUsed : 116 * 1024;
  static_assert(kSmem <= 232448, "exceeds the 227 KB shared memory of one sm_100 CTA");
};

// power-of-two factor t with max|t v| in [2^14, 2^15) for amax = max|v|:
// fp16 keeps its 11-bit significand over the largest entries and cannot
// overflow.  The exponent is capped at 126 so t stays finite (amax below
// 2^-112, subnormals included, gets t = 2^126 and max|t v| < 2^14); 1 for
// zero or non-finite amax.
__device__ __forceinline__ float pow2_scale(float amax) {
  const uint32_t b = __float_as_uint(amax);
  const int ex = (int)((b >> 23) & 0xFFu);
  if (!(amax > 0.0f) || ex == 0xFF) return 1.0f;
  return ldexpf(1.0f, min(14 - (ex - 127), 126));
}

// One or two streams (e.g. the keys and the values of an append), each
// with its own vectors, dictionary, codes and residual energies; the
// row tiles of stream 0 come first, then those of stream 1, so one launch
// spreads the tiles of both over the SMs.
struct TcParams {
  const void* x[2];
  int x_dtype;
  int64_t n_vec[2];
  const uint16_t* dict[2];
  int n;
  int k_atoms;
  uint32_t* codes[2];
  float* rsq[2];
  WsHeader* hdr;
  float* resid;        // [grid][D][kTileRows] fp32
  // dictionary statistics per stream: [0] max_i ||d_i||, [1] max_i
  // ||t d_i - fp16(t d_i)|| (f16 operands; 0 for bf16), [2] max_ij |d_ij| as
  // bits; t = dict_scale([2])
  const float* dmax[2];
  int tiles0;          // row tiles of stream 0
  int n_tiles;         // row tiles of both streams
  int n_atom_tiles;
};

// max(|a|, |b|) in one instruction (the sign of the result is the xor of
// the operands' signs; only its magnitude is used)
__device__ __forceinline__ float absmax2(float a, float b) {
  float r;
  asm("max.xorsign.abs.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
  return r;
}

// Instruction descriptor: D f32, A and B both f16 (F16=true) or both bf16,
// both K-major, N=128, M=128.
template <bool F16>
struct Idesc {
  static constexpr uint32_t value = (1u << 4) | ((F16 ? 0u : 1u) << 7) | ((F16 ? 0u : 1u) << 10) |
                                    ((uint32_t)(kAtomTile >> 3) << 17) |
                                    ((uint32_t)(kRows >> 4) << 24);
};

__device__ __forceinline__ float bf16_round(float v) {
  return __bfloat162float(__float2bfloat16_rn(v));
}

// ---- the kernel --------------------------------------------------------------
template <int D, bool F16>
__global__ void __launch_bounds__(kThreads, 1)
    encode_tc_kernel(const __grid_constant__ CUtensorMap tmap0,
                     const __grid_constant__ CUtensorMap tmap1, TcParams p) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_smem_1k(smem_raw);
  uint32_t* s_cw = reinterpret_cast<uint32_t*>(smem + C::kOffCw);
  float* s_best = reinterpret_cast<float*>(smem + C::kOffBest);
  uint32_t* s_cnt = reinterpret_cast<uint32_t*>(smem + C::kOffCnt);
  float* s_band = reinterpret_cast<float*>(smem + C::kOffBand);
  uint32_t* s_act = reinterpret_cast<uint32_t*>(smem + C::kOffAct);
  float* s_scl = reinterpret_cast<float*>(smem + C::kOffScl);
  float* s_fr = reinterpret_cast<float*>(smem + C::kOffFr);
  float* s_stg = reinterpret_cast<float*>(smem + C::kOffStg);
  float* s_rabs = reinterpret_cast<float*>(smem + C::kOffRes);
  uint32_t* s_ridx = reinterpret_cast<uint32_t*>(smem + C::kOffRes + kEpiThreads * 4);
  float* s_rcoef = reinterpret_cast<float*>(smem + C::kOffRes + kEpiThreads * 8);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile uint32_t* s_abort = misc + 0;
  volatile uint32_t* s_tmem = misc + 1;

  const uint32_t sB = smem_u32(smem);
  const uint32_t sA = smem_u32(smem + C::kOffA);
  auto bar_full = [&](int s) { return smem_u32(&bars[s]); };
  auto bar_empty = [&](int s) { return smem_u32(&bars[kStages + s]); };
  auto bar_tfull = [&](int b) { return smem_u32(&bars[2 * kStages + b]); };
  auto bar_tempty = [&](int b) { return smem_u32(&bars[2 * kStages + 2 + b]); };
  const uint32_t bar_afull = smem_u32(&bars[2 * kStages + 4]);
  const uint32_t bar_done = smem_u32(&bars[2 * kStages + 5]);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    *s_abort = 0u;
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar_full(s), 1);
      mbar_init(bar_empty(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar_tfull(b), 1);
      mbar_init(bar_tempty(b), kEpiWarps);
    }
    mbar_init(bar_afull, kLeadWarps);
    mbar_init(bar_done, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32((const void*)s_tmem)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;
  const int steps_total = p.k_atoms;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, last_phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < p.n_tiles; tile += gridDim.x)
        for (int j = 0; ok && j < steps_total; ++j)
          for (int a = 0; a < p.n_atom_tiles; ++a) {
            if (!mbar_wait(bar_empty(stage), phase ^ 1u, s_abort)) {
              ok = false;
              break;
            }
            mbar_expect_tx(bar_full(stage), (uint32_t)C::kStageBytes);
#pragma unroll
            for (int kb = 0; kb < C::KB; ++kb)
              tma_load_2d(sB + stage * C::kStageBytes + kb * (kAtomTile * 128),
                          tile < p.tiles0 ? &tmap0 : &tmap1, kb * 64, a * kAtomTile,
                          bar_full(stage));
            issued_mask |= 1u << stage;
            last_phase = (last_phase & ~(1u << stage)) | (phase << stage);
            if (++stage == kStages) {
              stage = 0;
              phase ^= 1u;
            }
          }
      if (!ok) {
        record_error(p.hdr, SDK_ERR_TIMEOUT, 0x40000000u | blockIdx.x);
        *s_abort = 1u;
      }
      // let every issued copy land before the CTA can exit
      for (int s = 0; s < kStages; ++s)
        if (issued_mask & (1u << s)) {
          uint32_t dummy = 0u;
          mbar_wait(bar_full(s), (last_phase >> s) & 1u, &dummy, 100000000ull);
        }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, tbuf = 0, tphase = 0, aphase = 0;
      bool ok = true;
      bool issued = false;
      for (int tile = blockIdx.x; ok && tile < p.n_tiles; tile += gridDim.x)
        for (int j = 0; ok && j < steps_total; ++j) {
          if (!mbar_wait(bar_afull, aphase, s_abort)) {
            ok = false;
            break;
          }
          aphase ^= 1u;
          tc_fence_after();
          for (int a = 0; a < p.n_atom_tiles; ++a) {
            if (!mbar_wait(bar_full(stage), phase, s_abort) ||
                !mbar_wait(bar_tempty(tbuf), tphase ^ 1u, s_abort)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t bbase = sB + stage * C::kStageBytes;
#pragma unroll
            for (int rs = 0; rs < kSets; ++rs) {
              const uint32_t d_tmem = tmem + tbuf * (kSets * kAtomTile) + rs * kAtomTile;
              const uint32_t abase = sA + rs * C::kABytes;
#pragma unroll
              for (int ks = 0; ks < C::KSTEPS; ++ks) {
                const uint32_t koff = (ks >> 2) * (kRows * 128) + (ks & 3) * 32;
                const uint32_t boff = (ks >> 2) * (kAtomTile * 128) + (ks & 3) * 32;
                tc_mma(d_tmem, smem_desc(abase + koff), smem_desc(bbase + boff), Idesc<F16>::value,
                       ks > 0 ? 1u : 0u);
              }
            }
            issued = true;
            tc_commit(bar_empty(stage));
            tc_commit(bar_tfull(tbuf));
            if (++stage == kStages) {
              stage = 0;
              phase ^= 1u;
            }
            tbuf ^= 1u;
            if (tbuf == 0u) tphase ^= 1u;
          }
        }
      if (!ok) {
        record_error(p.hdr, SDK_ERR_TIMEOUT, 0x41000000u | blockIdx.x);
        *s_abort = 1u;
      }
      if (issued) {
        // all MMAs of this thread complete before TMEM is released
        tc_commit(bar_done);
        uint32_t dummy = 0u;
        mbar_wait(bar_done, 0u, &dummy, 100000000ull);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // 16 warps: (row set, column half) x TMEM lane quarter.  Thread `tix`
    // scans 64 of the 128 columns of one residual row per atom tile; the
    // "lead" thread of the row (column half 0) merges both candidate lists
    // at the end of a step, picks, and updates the residual.
    // the current row tile's stream
    const uint16_t* cdict = p.dict[0];
    const float* cdmax = p.dmax[0];
    uint32_t* ccodes = p.codes[0];
    float* crsq = p.rsq[0];
    const int e = warp - 2;
    const int combo = e >> 2;
    const int rs = combo >> 1, half = combo & 1;
    const bool lead = half == 0;
    const int q = warp & 3;                   // TMEM lane quarter of this warp
    const int rin = q * 32 + lane;            // row within the set (TMEM lane)
    const int row = rs * kRows + rin;         // row within the tile
    const int tix = e * 32 + lane;            // partner (other half): tix ^ 128
    uint32_t* cw = s_cw + tix * kCand;
    float* stg = s_stg + e * 32;
    const unsigned lt = (1u << lane) - 1u;
    float* rres = p.resid + (int64_t)blockIdx.x * D * kTileRows + row;  // stride kTileRows
    float* fr = s_fr + (rs * 4 + (e & 3)) * D;                           // lead warps only
    // f16 operands: the MMA reads fp16(t d_i) for a power-of-two t, so a
    // tensor-core value approximates s t <r, d_i> for the row scale s; econv
    // is the largest conversion error ||t d_i - fp16(t d_i)|| and dmax bounds
    // the operand atom norms ||fp16(t d_i)||
    // (read where used, to keep them out of the scan loop's registers)
    auto tdict_of = [&] {
      return F16 ? pow2_scale(__int_as_float(__ldg(reinterpret_cast<const int*>(cdmax) + 2)))
                 : 1.0f;
    };
    uint8_t* arow = smem + C::kOffA + rs * C::kABytes + rin * 128;
    uint32_t tbuf = 0, tphase = 0;
    uint32_t n_rescored = 0;
    auto epi_sync = [] { asm volatile("bar.sync 1, %0;" ::"n"(kEpiThreads) : "memory"); };

    // A operand row: the residual times the row's power-of-two scale s,
    // rounded to the operand type.  Accumulates
    // the scaled rounding error ||s r - A||^2 and ||s r||^2.
    auto write_a_chunk = [&](int kc, const float (&r8)[8], float sc, float& e2, float& n2) {
      uint32_t w[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float a0 = r8[2 * u] * sc, a1 = r8[2 * u + 1] * sc;
        float b0, b1;
        if constexpr (F16) {
          const __half2 h = __floats2half2_rn(a0, a1);
          b0 = __low2float(h);
          b1 = __high2float(h);
          w[u] = *reinterpret_cast<const uint32_t*>(&h);
        } else {
          const __nv_bfloat162 h = __floats2bfloat162_rn(a0, a1);
          b0 = __low2float(h);
          b1 = __high2float(h);
          w[u] = *reinterpret_cast<const uint32_t*>(&h);
        }
        e2 = fmaf(a0 - b0, a0 - b0, e2);
        e2 = fmaf(a1 - b1, a1 - b1, e2);
        n2 = fmaf(a0, a0, n2);
        n2 = fmaf(a1, a1, n2);
      }
      const int kb = kc >> 3, c16 = kc & 7;
      uint4* dst = reinterpret_cast<uint4*>(arow + kb * (kRows * 128) + ((c16 ^ (rin & 7)) << 4));
      *dst = make_uint4(w[0], w[1], w[2], w[3]);
    };
    // row scale s of the A operand: exact, and for bf16 operands it keeps
    // the products of a tiny residual out of the fp32 subnormal range
    auto scale_of = [](float amax) { return pow2_scale(amax); };
    // writes the A row from the fp32 residual in rres; returns the band
    auto write_a_row = [&](float sc, float& n2_out) {
      float e2 = 0.0f, n2 = 0.0f;
#pragma unroll 1
      for (int kc = 0; kc < D / 8; ++kc) {
        float r8[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) r8[u] = rres[(kc * 8 + u) * kTileRows];
        write_a_chunk(kc, r8, sc, e2, n2);
      }
      n2_out = n2;
      // twice the bound on |c~ - s c| (scaled units): rounding of s r
      // (Cauchy-Schwarz with the largest operand atom norm), conversion of
      // the dictionary to the operand type, and slack for the accumulation
      const float econv = F16 ? __ldg(cdmax + 1) : 0.0f;
      const float dmax = __ldg(cdmax) * tdict_of() + econv;
      const float rn = sqrtf(n2);
      return 2.0f * dmax * sqrtf(e2) + 2.0f * econv * rn + 0.000244140625f * dmax * rn;
    };
    // fp32 correlation in k order (the CUDA-core encoder's arithmetic)
    auto dot_atom = [&](uint32_t i) {
      const uint4* dp = reinterpret_cast<const uint4*>(cdict + (int64_t)i * D);
      float sd = 0.0f;
#pragma unroll 4
      for (int kc = 0; kc < D / 8; ++kc) {
        const uint4 dv = __ldg(dp + kc);
        const uint32_t dw[4] = {dv.x, dv.y, dv.z, dv.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          sd = fmaf(rres[(kc * 8 + 2 * u) * kTileRows], bf16_lo(dw[u]), sd);
          sd = fmaf(rres[(kc * 8 + 2 * u + 1) * kTileRows], bf16_hi(dw[u]), sd);
        }
      }
      return sd;
    };
    // candidate word: bf16 of |c~| rounded up (order-preserving for
    // non-negative values) in the high half, atom index in the low half
    auto cand_val = [](uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); };

    for (int tile = blockIdx.x; tile < p.n_tiles; tile += gridDim.x) {
      const int sidx = tile < p.tiles0 ? 0 : 1;
      cdict = p.dict[sidx];
      cdmax = p.dmax[sidx];
      ccodes = p.codes[sidx];
      crsq = p.rsq[sidx];
      const void* cx = p.x[sidx];
      const int64_t grow = (int64_t)(tile - (sidx ? p.tiles0 : 0)) * kTileRows + row;
      const bool valid = grow < p.n_vec[sidx];
      if (lead && !*s_abort) {
        // residual <- x; A <- operand(scale * x)
        float amax = 0.0f;
#pragma unroll 1
        for (int kc = 0; kc < D / 8; ++kc) {
          float r8[8];
          if (valid) {
            if (p.x_dtype == SDK_F32) {
              const float4* xp = reinterpret_cast<const float4*>(
                  reinterpret_cast<const float*>(cx) + grow * D + kc * 8);
              const float4 xa = __ldg(xp), xb = __ldg(xp + 1);
              r8[0] = xa.x; r8[1] = xa.y; r8[2] = xa.z; r8[3] = xa.w;
              r8[4] = xb.x; r8[5] = xb.y; r8[6] = xb.z; r8[7] = xb.w;
            } else {
              const uint4 xv = __ldg(reinterpret_cast<const uint4*>(
                  reinterpret_cast<const uint16_t*>(cx) + grow * D + kc * 8));
              const uint32_t vw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                r8[2 * u] = bf16_lo(vw[u]);
                r8[2 * u + 1] = bf16_hi(vw[u]);
              }
            }
          } else {
#pragma unroll
            for (int u = 0; u < 8; ++u) r8[u] = 0.0f;
          }
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            rres[(kc * 8 + u) * kTileRows] = r8[u];
            amax = fmaxf(amax, fabsf(r8[u]));
          }
        }
        const float sc = scale_of(amax);
        float n2;
        s_band[row] = write_a_row(sc, n2);
        s_scl[row] = sc;
        s_act[row] = (valid && n2 > 0.0f) ? 1u : 0u;
        fence_proxy_async();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_afull);
      }
      epi_sync();
      float band = s_band[row];
      bool active = s_act[row] != 0u;

      float best_next = -INFINITY;   // lower bound on the next step's max
      for (int j = 0; j < steps_total; ++j) {
        float best = best_next, thr = best_next - band;
        best_next = -INFINITY;
        int cnt = 0;
        bool ovf = false;
#pragma unroll 1
        for (int a = 0; a < p.n_atom_tiles; ++a) {
          if (*s_abort) continue;
          // one lane waits so the warp stays converged for tcgen05.ld
          const bool got = lane == 0 ? mbar_wait(bar_tfull(tbuf), tphase, s_abort) : true;
          if (!__shfl_sync(0xffffffffu, got ? 1 : 0, 0)) {
            if (lane == 0) {
              record_error(p.hdr, SDK_ERR_TIMEOUT, 0x42000000u | blockIdx.x);
              *s_abort = 1u;
            }
            continue;
          }
          tc_fence_after();
          const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16) + tbuf * (kSets * kAtomTile) +
                                 rs * kAtomTile + half * 64;
          // two 32-column halves: 32 accumulator registers live at a time
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            uint32_t v[32];
            __syncwarp();  // reconverge (the previous half may have diverged)
            tmem_ld32(taddr + c * 32, v);
            tmem_ld_wait();
            if (c == 1) {
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(bar_tempty(tbuf));
            }
            // max |c~| of each 16-column group (balanced trees), then overall
            float m16[2];
#pragma unroll
            for (int g = 0; g < 2; ++g) {
              float t8[8];
#pragma unroll
              for (int i = 0; i < 8; ++i)
                t8[i] = absmax2(__uint_as_float(v[g * 16 + i]), __uint_as_float(v[g * 16 + i + 8]));
#pragma unroll
              for (int i = 0; i < 4; ++i) t8[i] = absmax2(t8[i], t8[i + 4]);
              m16[g] = fabsf(absmax2(absmax2(t8[0], t8[2]), absmax2(t8[1], t8[3])));
            }
            const float mt = fmaxf(m16[0], m16[1]);
            const bool trig = active && mt >= thr;
            if (trig) {
              best = fmaxf(best, mt);
              thr = best - band;
            }
            // Candidates: every column within `band` of the running maximum.
            // Triggering lanes stage their raw 16-column groups in shared
            // memory, two at a time; each half-warp tests and appends one
            // staged group to its owner's list.
            if (__ballot_sync(0xffffffffu, trig) == 0u) continue;
            const int col0 = a * kAtomTile + half * 64 + c * 32;
#pragma unroll
            for (int g = 0; g < 2; ++g) {
              unsigned tm = __ballot_sync(0xffffffffu, trig && m16[g] >= thr);
              while (tm != 0u) {
                const int L1 = __ffs(tm) - 1;
                tm &= tm - 1u;
                const int L2 = tm != 0u ? __ffs(tm) - 1 : -1;
                if (L2 >= 0) tm &= tm - 1u;
                if (lane == L1 || lane == L2) {
                  uint4* s4 = reinterpret_cast<uint4*>(stg + (lane == L1 ? 0 : 16));
#pragma unroll
                  for (int i = 0; i < 4; ++i)
                    s4[i] = make_uint4(v[g * 16 + 4 * i], v[g * 16 + 4 * i + 1],
                                       v[g * 16 + 4 * i + 2], v[g * 16 + 4 * i + 3]);
                }
                __syncwarp();
                const int hl = lane >> 4;                    // half-warp -> owner
                const int L = hl == 0 ? L1 : L2;
                const int Ls = L < 0 ? L1 : L;               // valid shuffle source
                const float thrL = __shfl_sync(0xffffffffu, thr, Ls);
                const int cntL0 = __shfl_sync(0xffffffffu, cnt, Ls);
                const float av = fabsf(stg[lane]);
                const int col = col0 + g * 16 + (lane & 15);
                const bool take = L >= 0 && av >= thrL && col < p.n;
                const unsigned pm = __ballot_sync(0xffffffffu, take);
                const unsigned pmh = hl == 0 ? (pm & 0xFFFFu) : (pm >> 16);
                const int np = __popc(pmh);
                int cntL = cntL0;
                const bool full = L >= 0 && cntL + np > kCand;
                if (__ballot_sync(0xffffffffu, full) != 0u) {
                  // make room: owners drop their stale candidates
                  if (lane == L1 || lane == L2) {
                    int w = 0;
                    for (int t = 0; t < cnt; ++t)
                      if (cand_val(cw[t]) >= thr) cw[w++] = cw[t];
                    cnt = w;
                  }
                  __syncwarp();
                  cntL = __shfl_sync(0xffffffffu, cnt, Ls);
                }
                if (take) {
                  const int pos = cntL + __popc(pmh & ((1u << (lane & 15)) - 1u));
                  const uint32_t ab = __float_as_uint(av);
                  if (pos < kCand)
                    s_cw[(e * 32 + L) * kCand + pos] =
                        (((ab + 0xFFFFu) >> 16) << 16) | (uint32_t)col;
                }
                const int np1 = __popc(pm & 0xFFFFu), np2 = __popc(pm >> 16);
                const int cn1 = __shfl_sync(0xffffffffu, cntL, 0);
                const int cn2 = __shfl_sync(0xffffffffu, cntL, 16);
                if (lane == L1) {
                  ovf |= cn1 + np1 > kCand;
                  cnt = min(cn1 + np1, kCand);
                } else if (lane == L2) {
                  ovf |= cn2 + np2 > kCand;
                  cnt = min(cn2 + np2, kCand);
                }
                __syncwarp();
              }
            }
          }
          tbuf ^= 1u;
          if (tbuf == 0u) tphase ^= 1u;
        }

        // ---- step end: merge the two halves of every row, pick, update
        s_best[tix] = best;
        s_cnt[tix] = (uint32_t)cnt | (ovf ? 0x80000000u : 0u);
        epi_sync();
        const float pbest = s_best[tix ^ 128];
        const uint32_t pcw_cnt = s_cnt[tix ^ 128];
        uint32_t sidx = 0xFFFFFFFFu, own_best = 0xFFFFFFFFu;   // own top-2 candidates
        const bool anyovf = ovf || (pcw_cnt >> 31) != 0u;
        {
          // each thread re-scores its own candidates that survive the row's
          // threshold; the chunk-outer loop reads the fp32 residual once for
          // all of them and keeps every dot in k order
          const float gthr = fmaxf(best, pbest) - band;
          float babs = -1.0f, bcoef = 0.0f, sabs = -1.0f;
          uint32_t bidx = 0xFFFFFFFFu;
          sidx = 0xFFFFFFFFu;
          if (active && !anyovf && !*s_abort) {
            bool ok_e[kCand];
            uint32_t ix[kCand];
            float acc[kCand];
#pragma unroll
            for (int e2 = 0; e2 < kCand; ++e2) {
              const uint32_t wv = cw[e2];
              ok_e[e2] = e2 < cnt && cand_val(wv) >= gthr;
              ix[e2] = wv & 0x7FFFu;
              acc[e2] = 0.0f;
              n_rescored += ok_e[e2] ? 1u : 0u;
            }
#pragma unroll 1
            for (int kc = 0; kc < D / 8; ++kc) {
              float r8[8];
#pragma unroll
              for (int u = 0; u < 8; ++u) r8[u] = rres[(kc * 8 + u) * kTileRows];
#pragma unroll
              for (int e2 = 0; e2 < kCand; ++e2) {
                if (!ok_e[e2]) continue;
                const uint4 dv = __ldg(reinterpret_cast<const uint4*>(cdict + (int64_t)ix[e2] * D) + kc);
                float sd = acc[e2];
                sd = fmaf(r8[0], bf16_lo(dv.x), sd);
                sd = fmaf(r8[1], bf16_hi(dv.x), sd);
                sd = fmaf(r8[2], bf16_lo(dv.y), sd);
                sd = fmaf(r8[3], bf16_hi(dv.y), sd);
                sd = fmaf(r8[4], bf16_lo(dv.z), sd);
                sd = fmaf(r8[5], bf16_hi(dv.z), sd);
                sd = fmaf(r8[6], bf16_lo(dv.w), sd);
                sd = fmaf(r8[7], bf16_hi(dv.w), sd);
                acc[e2] = sd;
              }
            }
#pragma unroll
            for (int e2 = 0; e2 < kCand; ++e2) {
              if (!ok_e[e2]) continue;
              const float aa = fabsf(acc[e2]);
              if (aa > babs || (aa == babs && ix[e2] < bidx)) {
                sabs = babs;
                sidx = bidx;
                babs = aa;
                bcoef = acc[e2];
                bidx = ix[e2];
              } else if (aa > sabs || (aa == sabs && ix[e2] < sidx)) {
                sabs = aa;
                sidx = ix[e2];
              }
            }
          }
          own_best = bidx;
          s_rabs[tix] = babs;
          s_ridx[tix] = bidx;
          s_rcoef[tix] = bcoef;
        }
        epi_sync();
        if (lead && !*s_abort) {
          uint32_t pick = 0u;
          float coef = 0.0f;
          if (active && !anyovf) {
            // the better of the two halves' picks (ties: lower atom index)
            float babs = s_rabs[tix];
            uint32_t bidx = s_ridx[tix];
            coef = s_rcoef[tix];
            const float oabs = s_rabs[tix ^ 128];
            const uint32_t oidx = s_ridx[tix ^ 128];
            if (oabs > babs || (oabs == babs && oidx < bidx)) {
              babs = oabs;
              bidx = oidx;
              coef = s_rcoef[tix ^ 128];
            }
            s_ridx[tix] = bidx;   // the row's pick, read by the partner after the barrier
            if (bidx < (uint32_t)p.n) {
              pick = bidx;
            } else {
              // no candidate survived (only possible with non-finite
              // correlations): keep atom 0 with coefficient 0 and report it
              record_error(p.hdr, SDK_ERR_DEVICE_CHECK, 0x43000000u | (uint32_t)j);
              pick = 0u;
              coef = 0.0f;
            }
          }
          // rows whose candidate list overflowed: exact fp32 scan of every
          // atom shared by the warp, one such row at a time
          uint32_t ovm = __ballot_sync(0xffffffffu, active && anyovf);
          if (ovm != 0u && lane == 0) atomicAdd(&p.hdr->enc_fallback, (uint32_t)__popc(ovm));
#pragma unroll 1
          while (ovm != 0u) {
            const int src = __ffs(ovm) - 1;
            ovm &= ovm - 1u;
            const float* rsrc = p.resid + (int64_t)blockIdx.x * D * kTileRows +
                                (rs * kRows + q * 32 + src);
            for (int k = lane; k < D; k += 32) fr[k] = rsrc[k * kTileRows];
            __syncwarp();
            float bab = -1.0f, bc = 0.0f;
            uint32_t bi = 0u;
#pragma unroll 1
            for (int i = lane; i < p.n; i += 32) {
              const uint4* dp = reinterpret_cast<const uint4*>(cdict + (int64_t)i * D);
              float sd = 0.0f;
#pragma unroll 4
              for (int kc = 0; kc < D / 8; ++kc) {
                const uint4 dv = __ldg(dp + kc);
                const float4 ra = *reinterpret_cast<const float4*>(fr + kc * 8);
                const float4 rb = *reinterpret_cast<const float4*>(fr + kc * 8 + 4);
                sd = fmaf(ra.x, bf16_lo(dv.x), sd);
                sd = fmaf(ra.y, bf16_hi(dv.x), sd);
                sd = fmaf(ra.z, bf16_lo(dv.y), sd);
                sd = fmaf(ra.w, bf16_hi(dv.y), sd);
                sd = fmaf(rb.x, bf16_lo(dv.z), sd);
                sd = fmaf(rb.y, bf16_hi(dv.z), sd);
                sd = fmaf(rb.z, bf16_lo(dv.w), sd);
                sd = fmaf(rb.w, bf16_hi(dv.w), sd);
              }
              if (fabsf(sd) > bab) {
                bab = fabsf(sd);
                bc = sd;
                bi = (uint32_t)i;
              }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
              const float oa = __shfl_xor_sync(0xffffffffu, bab, o);
              const float oc = __shfl_xor_sync(0xffffffffu, bc, o);
              const uint32_t oi = __shfl_xor_sync(0xffffffffu, bi, o);
              if (oa > bab || (oa == bab && oi < bi)) {
                bab = oa;
                bc = oc;
                bi = oi;
              }
            }
            if (lane == src) {
              coef = bc;
              pick = bi;
            }
            __syncwarp();
          }
          if (pick >= (uint32_t)p.n) {
            record_error(p.hdr, SDK_ERR_DEVICE_CHECK, 0x44000000u | pick);
            pick = 0u;
            coef = 0.0f;
          }
          if (valid) ccodes[grow * p.k_atoms + j] = make_word(coef, pick);

          // residual update r -= coef * d_pick; next A operand
          if (active) {
            float amax = 0.0f;
            const uint4* dp = reinterpret_cast<const uint4*>(cdict + (int64_t)pick * D);
#pragma unroll 1
            for (int kc = 0; kc < D / 8; ++kc) {
              const uint4 dv = __ldg(dp + kc);
              const uint32_t dw[4] = {dv.x, dv.y, dv.z, dv.w};
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                float* r0 = rres + (kc * 8 + 2 * u) * kTileRows;
                float* r1 = rres + (kc * 8 + 2 * u + 1) * kTileRows;
                const float n0 = fmaf(-coef, bf16_lo(dw[u]), *r0);
                const float n1 = fmaf(-coef, bf16_hi(dw[u]), *r1);
                *r0 = n0;
                *r1 = n1;
                amax = fmaxf(amax, fmaxf(fabsf(n0), fabsf(n1)));
              }
            }
            if (j + 1 < steps_total) {
              const float sc = scale_of(amax);
              float n2;
              s_band[row] = write_a_row(sc, n2);
              s_scl[row] = sc;
              s_act[row] = n2 > 0.0f ? 1u : 0u;
            }
          }
          if (j + 1 < steps_total) {
            fence_proxy_async();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_afull);
          }
        }
        epi_sync();
        band = s_band[row];
        active = s_act[row] != 0u;
        // lower bound for the next step: the fp32 correlation of the new
        // residual with this thread's best candidate that was not picked;
        // |c'| - band/2 never exceeds that atom's tensor-core value, hence
        // the next step's maximum (band/2 covers the rounding and
        // accumulation errors)
        if (active && !anyovf && j + 1 < steps_total && !*s_abort) {
          const uint32_t pick_row = s_ridx[lead ? tix : (tix ^ 128)];
          const uint32_t ru = own_best != pick_row ? own_best : sidx;
          if (ru < (uint32_t)p.n) best_next = fabsf(dot_atom(ru)) * s_scl[row] * tdict_of() - 0.5f * band;
        }
      }
      if (lead && valid && crsq != nullptr && !*s_abort) {
        float sq = 0.0f;
        for (int k = 0; k < D; ++k) {
          const float r = rres[k * kTileRows];
          sq = fmaf(r, r, sq);
        }
        crsq[grow] = sq;
      }
    }
    n_rescored = __reduce_add_sync(0xffffffffu, n_rescored);
    if (lane == 0 && n_rescored) atomicAdd(&p.hdr->enc_cands, n_rescored);
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kTmemCols)
                 : "memory");
  }
}

// Dictionary statistics, one thread per atom (16-byte loads): st[0] =
// max_i ||d_i||, st[2] = max_ij |d_ij| (float bits; both maxima via integer
// atomicMax, valid for non-negative floats).  st must be zero before the
// launch.
template <int D>
__global__ void __launch_bounds__(128) dict_stats_kernel(const uint16_t* dict, int n, float* st) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  float s = 0.0f, am = 0.0f;
  if (i < n) {
    const uint4* dp = reinterpret_cast<const uint4*>(dict + (int64_t)i * D);
#pragma unroll
    for (int kc = 0; kc < D / 8; ++kc) {
      const uint4 v = __ldg(dp + kc);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float lo = bf16_lo(w[u]), hi = bf16_hi(w[u]);
        s = fmaf(lo, lo, s);
        s = fmaf(hi, hi, s);
        am = fmaxf(am, fmaxf(fabsf(lo), fabsf(hi)));
      }
    }
  }
  float m = sqrtf(s);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
  }
  if ((threadIdx.x & 31) == 0) {
    if (m > 0.0f) atomicMax(reinterpret_cast<int*>(st), __float_as_int(m));
    if (am > 0.0f) atomicMax(reinterpret_cast<int*>(st) + 2, __float_as_int(am));
  }
}

// fp16 operand copy of the dictionary: out = fp16(t d) with t from st[2];
// st[1] = max_i ||t d_i - fp16(t d_i)|| (zero before the launch)
template <int D>
__global__ void __launch_bounds__(128) dict_f16_kernel(const uint16_t* dict, int n, float* st,
                                                       __half* out) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  const float t = pow2_scale(__int_as_float(reinterpret_cast<const int*>(st)[2]));
  float e = 0.0f;
  if (i < n) {
    const uint4* dp = reinterpret_cast<const uint4*>(dict + (int64_t)i * D);
    uint4* op = reinterpret_cast<uint4*>(out + (int64_t)i * D);
#pragma unroll
    for (int kc = 0; kc < D / 8; ++kc) {
      const uint4 v = __ldg(dp + kc);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
      uint32_t o[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float lo = bf16_lo(w[u]) * t, hi = bf16_hi(w[u]) * t;
        const __half2 h = __floats2half2_rn(lo, hi);
        const float dl = lo - __low2float(h), dh = hi - __high2float(h);
        e = fmaf(dl, dl, e);
        e = fmaf(dh, dh, e);
        o[u] = *reinterpret_cast<const uint32_t*>(&h);
      }
      op[kc] = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
  float m = sqrtf(e);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0 && m > 0.0f) atomicMax(reinterpret_cast<int*>(st) + 1, __float_as_int(m));
}

// operand type of the tensor-core encoder: fp16 (default) or bf16 when the
// environment variable SDK_ENCODE_OPERANDS is "bf16"
bool operands_f16() {
  static int mode = -1;
  if (mode < 0) {
    const char* v = getenv("SDK_ENCODE_OPERANDS");
    mode = (v != nullptr && strcmp(v, "bf16") == 0) ? 0 : 1;
  }
  return mode == 1;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000,
                                         cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

}  // namespace tc

// scratch: 256 B of dictionary statistics per stream, the fp16 operand
// copy of every stream's dictionary (256-byte aligned), then one fp32
// residual tile per CTA
static size_t dict_copy_bytes(int head_dim, int n_atoms) {
  return ((size_t)n_atoms * head_dim * 2 + 255) & ~(size_t)255;
}

size_t encode_tc_scratch_bytes(int64_t n_vec, int head_dim, int n_atoms, int streams) {
  if ((head_dim != 64 && head_dim != 128) || n_vec <= 0) return 256;
  int64_t tiles = (n_vec + tc::kTileRows - 1) / tc::kTileRows + (streams - 1);
  if (tiles > tc::kMaxCtas) tiles = tc::kMaxCtas;
  return (size_t)streams * (256 + dict_copy_bytes(head_dim, n_atoms)) +
         (size_t)tiles * head_dim * tc::kTileRows * 4;
}

sdk_status launch_encode_tc(const EncodeParams* ps, int streams, int head_dim, void* scratch,
                            size_t scratch_bytes, cudaStream_t stream, bool* taken) {
  *taken = false;
  if (head_dim != 64 && head_dim != 128) return SDK_OK;
  if (streams < 1 || streams > 2) return SDK_OK;
  if (streams == 2 && (ps[1].n != ps[0].n || ps[1].k_atoms != ps[0].k_atoms ||
                       ps[1].x_dtype != ps[0].x_dtype))
    return SDK_OK;
  int64_t tiles_s[2] = {0, 0};
  for (int s = 0; s < streams; ++s) {
    if (ps[s].n_vec <= 0) return SDK_OK;
    // vectorised 16-byte loads of x rows need a 16-byte aligned x
    if ((reinterpret_cast<uintptr_t>(ps[s].x) & 15u) != 0u) return SDK_OK;
    tiles_s[s] = (ps[s].n_vec + tc::kTileRows - 1) / tc::kTileRows;
  }
  auto fn = tc::encode_fn();
  if (fn == nullptr) return SDK_OK;  // no driver entry point: CUDA-core path
  const EncodeParams& p = ps[0];
  const int64_t tiles = tiles_s[0] + tiles_s[1];
  int64_t grid = tiles;
  const int sms = num_sms();
  if (grid > sms) grid = sms;
  if (grid > tc::kMaxCtas) grid = tc::kMaxCtas;
  const bool f16 = tc::operands_f16();
  const size_t per_cta = (size_t)head_dim * tc::kTileRows * 4;
  const size_t dict_bytes = dict_copy_bytes(head_dim, p.n);
  const size_t per_stream = 256 + dict_bytes;
  if (scratch_bytes < (size_t)streams * per_stream + (size_t)grid * per_cta) return SDK_ERR_CAPACITY;

  CUtensorMap maps[2];
  float* stats[2];
  __half* dict16[2];
  for (int s = 0; s < streams; ++s) {
    char* base_s = reinterpret_cast<char*>(scratch) + (size_t)s * per_stream;
    stats[s] = reinterpret_cast<float*>(base_s);
    dict16[s] = reinterpret_cast<__half*>(base_s + 256);
    const cuuint64_t dims[2] = {(cuuint64_t)head_dim, (cuuint64_t)p.n};
    const cuuint64_t strides[1] = {(cuuint64_t)head_dim * 2};
    const cuuint32_t box[2] = {64u, (cuuint32_t)tc::kAtomTile};
    const cuuint32_t estr[2] = {1u, 1u};
    void* base = f16 ? static_cast<void*>(dict16[s]) : const_cast<uint16_t*>(ps[s].dict);
    CUresult cr = fn(&maps[s], f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                     2, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (cr != CUDA_SUCCESS) return SDK_ERR_INVALID_ARG;
  }
  if (streams == 1) maps[1] = maps[0];
  *taken = true;

  const unsigned dgrid = (unsigned)((p.n + 127) / 128);
  for (int s = 0; s < streams; ++s) {
    if (cudaMemsetAsync(stats[s], 0, 4 * sizeof(float), stream) != cudaSuccess) return SDK_ERR_CUDA;
    if (head_dim == 128) {
      tc::dict_stats_kernel<128><<<dgrid, 128, 0, stream>>>(ps[s].dict, p.n, stats[s]);
      if (f16) tc::dict_f16_kernel<128><<<dgrid, 128, 0, stream>>>(ps[s].dict, p.n, stats[s], dict16[s]);
    } else {
      tc::dict_stats_kernel<64><<<dgrid, 128, 0, stream>>>(ps[s].dict, p.n, stats[s]);
      if (f16) tc::dict_f16_kernel<64><<<dgrid, 128, 0, stream>>>(ps[s].dict, p.n, stats[s], dict16[s]);
    }
  }

  tc::TcParams tp;
  for (int s = 0; s < 2; ++s) {
    const int u = s < streams ? s : 0;
    tp.x[s] = ps[u].x;
    tp.n_vec[s] = s < streams ? ps[s].n_vec : 0;
    tp.dict[s] = ps[u].dict;
    tp.codes[s] = ps[u].codes;
    tp.rsq[s] = ps[u].rsq;
    tp.dmax[s] = stats[u];
  }
  tp.x_dtype = p.x_dtype;
  tp.n = p.n;
  tp.k_atoms = p.k_atoms;
  tp.hdr = p.hdr;
  tp.resid = reinterpret_cast<float*>(reinterpret_cast<char*>(scratch) + (size_t)streams * per_stream);
  tp.tiles0 = (int)tiles_s[0];
  tp.n_tiles = (int)tiles;
  tp.n_atom_tiles = (p.n + tc::kAtomTile - 1) / tc::kAtomTile;

  static unsigned long long attr_set = 0ull;
  if (device_needs_setup(&attr_set)) {
    cudaFuncSetAttribute(tc::encode_tc_kernel<128, true>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, tc::Cfg<128>::kSmem);
    cudaFuncSetAttribute(tc::encode_tc_kernel<64, true>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, tc::Cfg<64>::kSmem);
    cudaFuncSetAttribute(tc::encode_tc_kernel<128, false>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, tc::Cfg<128>::kSmem);
    cudaFuncSetAttribute(tc::encode_tc_kernel<64, false>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, tc::Cfg<64>::kSmem);
    device_setup_done(&attr_set);
  }
  const dim3 g((unsigned)grid);
  cudaEvent_t t0 = nullptr, t1 = nullptr;
  timing_slot(&t0, &t1);
  if (t0 != nullptr && timing_record(t0, stream) != cudaSuccess) return SDK_ERR_CUDA;
  if (head_dim == 128) {
    if (f16)
      tc::encode_tc_kernel<128, true><<<g, tc::kThreads, tc::Cfg<128>::kSmem, stream>>>(maps[0], maps[1], tp);
    else
      tc::encode_tc_kernel<128, false><<<g, tc::kThreads, tc::Cfg<128>::kSmem, stream>>>(maps[0], maps[1], tp);
  } else {
    if (f16)
      tc::encode_tc_kernel<64, true><<<g, tc::kThreads, tc::Cfg<64>::kSmem, stream>>>(maps[0], maps[1], tp);
    else
      tc::encode_tc_kernel<64, false><<<g, tc::kThreads, tc::Cfg<64>::kSmem, stream>>>(maps[0], maps[1], tp);
  }
  if (t1 != nullptr && timing_record(t1, stream) != cudaSuccess) return SDK_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? SDK_OK : SDK_ERR_CUDA;
}

}  // namespace sdk
