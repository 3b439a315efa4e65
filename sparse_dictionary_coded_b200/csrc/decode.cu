// Decode attention over dictionary codes with query-aware hierarchical
// sparsity ("LLM Inference in a Flash!", evolve.pub review, Summary: score
// all tokens with Klow=3 atoms, refine the top 10% with Khigh=16; FAQ on the
// 15x compression: only 3 atoms score most tokens).
//
// One layer, B sequences, R = B*Hq query heads.  Kernels, in stream order:
//   qd_tc_kernel     (qd_tc.cu) QD[r][a] = <q_r, D_K[a]> on the tensor cores,
//                    and zeroes the per-head selection state, histograms
//                    and `out`; qd_kernel here is the fp32 CUDA-core form.
//   klow_kernel      s_lo for every token from the 3 k_lo planes (12 B per
//                    token, coalesced) and QD staged in shared memory;
//                    writes order-preserving keys and the 12-bit radix
//                    histogram of every head.
//   pass2_kernel     finds the histogram bucket of the k-th key; tokens
//                    above it are selected, tokens inside it become
//                    candidates (compacted, with a second 12-bit histogram),
//                    tokens below go to the complement.
//   final_kernel     one CTA per head: last radix digits over the
//                    candidates, the exact k-th key, tie handling by token
//                    index, and the rest of the selected set.
//   attend_kernel    s_t = scale * sum_{j<khigh} c_tj QD[idx_tj] for the
//                    selected tokens (64-byte k_full records), p = softmax,
//                    and the scatter w[idx^V_tj] += p_t c^V_tj into a
//                    shared-memory per-atom weight tile (fixed-point
//                    atomics); one cluster of CTAs per head shares the
//                    softmax statistics and sums its tiles through
//                    distributed shared memory into w (three bf16 parts).
//   out_tc_kernel    (out_tc.cu) out += w D_V on the tensor cores; out_kernel
//                    here is the fp32 CUDA-core form.
// The Klow scan and pass 2 split the layer's tokens over their CTAs with a
// start-up cost charged per head (for_segments).
#include <cooperative_groups.h>
#include <stdio.h>
#include <stdlib.h>
#include <atomic>
#include <mutex>
#include <type_traits>

#include "sdk_internal.cuh"

namespace sdk {


// Work split over the heads of a layer.  A CTA pays a fixed start-up for
// every head it touches (staging, histogram search, flush, pipeline fill)
// on top of a cost per token, so the token range is split uniformly over a
// virtual space in which each head of sequence b spans `a` start-up units
// and then its cnt[b] tokens: a CTA that crosses into another head takes
// `a` fewer tokens.  off[b] = sum_{b' < b} Hq * cnt[b'] (real tokens);
// head (b, h) starts at virtual position off[b] + a*Hq*b + h*(cnt[b] + a).
__device__ __forceinline__ int64_t virtual_total(const int64_t* off, int B, int Hq, int64_t a) {
  return off[B] + a * Hq * (int64_t)B;
}

// Walks this CTA's share [V0, V1) of the virtual space: f(b, h, i0, i1) is
// called with block-uniform arguments for every head whose tokens
// [i0, i1) (i1 > i0) fall in the share.
template <class F>
__device__ __forceinline__ void for_segments(const int64_t* off, const int* cnt, int B, int Hq,
                                             int64_t a, F f) {
  const int64_t VT = virtual_total(off, B, Hq, a);
  const int64_t V0 = VT * blockIdx.x / gridDim.x;
  const int64_t V1 = VT * (blockIdx.x + 1) / gridDim.x;
  int64_t V = V0;
  int b = 0;
  while (V < V1) {
    while (b + 1 < B && off[b + 1] + a * Hq * (int64_t)(b + 1) <= V) ++b;
    const int64_t vb = off[b] + a * Hq * (int64_t)b;
    const int64_t hl = (int64_t)cnt[b] + a;           // virtual length of one head
    const int64_t local = V - vb;
    const int h = (int)(local / hl);
    const int64_t hs = vb + (int64_t)h * hl;          // virtual start of head h
    const int64_t e = min(V1, hs + hl);
    const int64_t i0 = max(V - hs - a, (int64_t)0);
    const int64_t i1 = e - hs - a;
    if (i1 > i0) f(b, h, i0, i1);
    V = e;
  }
}

// Block-wide search over NB histogram bins taken from the highest bin down:
// the bin holding the k-th element (1-based), the count in higher bins and
// the count in that bin.  s_tmp: >= 40 words of shared memory.  Sets
// *bad when k is 0 or exceeds the histogram total.
template <int NB, bool kL2 = false>   // kL2: hist is global memory written by other CTAs
__device__ void block_find_desc(const uint32_t* hist, uint32_t k,
                                uint32_t* s_tmp, uint32_t& bin,
                                uint32_t& above, uint32_t& cnt, bool& bad) {
  constexpr int PER = (NB + 511) / 512;
  const int tid = threadIdx.x;
  if (tid == 0) {
    s_tmp[32] = 0u;
    s_tmp[33] = 0u;
    s_tmp[34] = 0u;
    s_tmp[35] = 1u;
  }
  uint32_t c[PER];
  uint32_t sum = 0;
#pragma unroll
  for (int u = 0; u < PER; ++u) {
    const int rb = tid * PER + u;
    c[u] = rb < NB ? (kL2 ? __ldcg(hist + NB - 1 - rb) : hist[NB - 1 - rb]) : 0u;
    sum += c[u];
  }
  uint32_t tot;
  const uint32_t incl = block_incl_scan(sum, s_tmp, &tot);
  const uint32_t excl = incl - sum;
  if (k >= 1u && excl < k && k <= incl) {
    uint32_t acc = excl;
#pragma unroll
    for (int u = 0; u < PER; ++u) {
      if (acc < k && acc + c[u] >= k) {
        s_tmp[32] = (uint32_t)(NB - 1 - (tid * PER + u));
        s_tmp[33] = acc;
        s_tmp[34] = c[u];
        s_tmp[35] = 0u;
      }
      acc += c[u];
    }
  }
  __syncthreads();
  bin = s_tmp[32];
  above = s_tmp[33];
  cnt = s_tmp[34];
  bad = s_tmp[35] != 0u;
  __syncthreads();
}

constexpr int kTable = 32768;   // shared QD / weight tables: every 15-bit index

// ---------------------------------------------------------------- qd_kernel
// QD[r][a] = sum_k q[r][k] D_K[a][k].  A CTA takes kGvTiles atom tiles of
// kGvAtoms atoms and RB row blocks of 32 query rows (1 x 1 for up to 32
// rows, 4 x 2 above); two warps per (tile, row block).  Every atom tile of the CTA is requested at once with
// cp.async (bf16 [atom][D], the 16-byte chunks of atom a XOR-swizzled by
// a & 7), so the CTA's whole share of the dictionary is in flight before the
// first FMA; the query rows are staged fp32 [k][32] (4-row groups
// XOR-swizzled by k).  Lane (ta, tr) of warp w of a pair owns atoms
// 32w + ta + 8x (x = 0..3) and rows 8tr .. 8tr+7: per 8 values of k, four
// 16-byte atom loads (conflict-free through the swizzle) and sixteen
// broadcast row loads feed 256 FMAs (fp32, k order).
// The first kernel of a call also zeroes the per-head selection state, both
// histograms and `out` (accumulated with reductions by out_kernel).
constexpr int kGvAtoms = 64;

__device__ __forceinline__ int qswz(int k, int r) { return (((r >> 2) ^ (k & 7)) << 2) | (r & 3); }

constexpr int qd_smem_bytes(int d, int rb, int tiles) { return tiles * kGvAtoms * d * 2 + rb * d * 32 * 4; }

template <int D, int RB, int kGvTiles>
__global__ void __launch_bounds__(64 * kGvTiles * RB, (RB > 1 ? 2 : 1)) qd_kernel(DecodeParams p) {
  pdl_wait();     // nothing global is touched before the previous kernel is done
  pdl_launch();
  constexpr int kThreads = 64 * kGvTiles * RB;
  constexpr int kChunks = D / 8;                  // 16-byte chunks per atom row
  extern __shared__ uint4 qd_smem[];
  uint4* Dt = qd_smem;                            // [tile][atom][chunk]
  float* Qs = reinterpret_cast<float*>(qd_smem + kGvTiles * kGvAtoms * kChunks);  // [rb][k][32]
  const int n = p.n, R = p.R, tid = threadIdx.x;
  const int a0 = blockIdx.x * (kGvTiles * kGvAtoms);
  const int r0 = blockIdx.y * (32 * RB);
  // dictionary tiles: every chunk of the CTA in flight at once
  for (int e = tid; e < kGvTiles * kGvAtoms * kChunks; e += kThreads) {
    const int a = e / kChunks, c = e % kChunks;   // a: atom within the CTA
    const bool v = a0 + a < n;
    const uint4* src = reinterpret_cast<const uint4*>(p.dk + (int64_t)(v ? a0 + a : 0) * D) + c;
    cp_async16(Dt + a * kChunks + (c ^ (a & 7)), src, v);
  }
  cp_async_commit();
  {
    const int64_t nthr = (int64_t)gridDim.x * gridDim.y * kThreads;
    const int64_t g0 = ((int64_t)blockIdx.y * gridDim.x + blockIdx.x) * kThreads + tid;
    const int64_t hwords = p.bracket ? 0 : (int64_t)R * 4096;   // radix selection path only
    for (int64_t e = g0; e < hwords; e += nthr) {
      p.hist1[e] = 0u;
      p.hist2[e] = 0u;
    }
    for (int64_t e = g0; e < (int64_t)R * D; e += nthr) p.out[e] = 0.0f;
    for (int64_t e = g0; e < (int64_t)R; e += nthr) {
      sdk_select_state st = {};
      st.k = (uint32_t)p.kcnt[e / p.Hq];
      p.st[e] = st;
    }
  }
  // query rows (16-byte loads along k, all of a thread's loads in flight
  // before its first store)
  constexpr int kQ4 = RB * 32 * (D / 4);
  constexpr int kQPer = (kQ4 + kThreads - 1) / kThreads;
  for (int e0 = tid; e0 < kQ4; e0 += kQPer * kThreads) {
    float4 v[kQPer];
#pragma unroll
    for (int u = 0; u < kQPer; ++u) {
      const int e = e0 + u * kThreads;
      const int k4 = e % (D / 4), rr = e / (D / 4);
      v[u] = (e < kQ4 && r0 + rr < R)
                 ? __ldg(reinterpret_cast<const float4*>(p.q + (int64_t)(r0 + rr) * D) + k4)
                 : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < kQPer; ++u) {
      const int e = e0 + u * kThreads;
      if (e >= kQ4) break;
      const int k4 = e % (D / 4), rr = e / (D / 4);
      const int rb = rr >> 5, r = rr & 31;
      float* qb = Qs + rb * D * 32;
      const float x[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
      for (int j = 0; j < 4; ++j) qb[(4 * k4 + j) * 32 + qswz(4 * k4 + j, r)] = x[j];
    }
  }
  cp_async_wait<0>();
  __syncthreads();
  const int lane = tid & 31, warp = tid >> 5;
  const int pair = warp >> 1, wp = warp & 1;
  const int tile = pair % kGvTiles, rb = pair / kGvTiles;
  const int ta = lane & 7, tr = lane >> 3;
  const uint4* Dtile = Dt + tile * kGvAtoms * kChunks;
  const float* Qb = Qs + rb * D * 32;
  float acc[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int x = 0; x < 4; ++x) acc[i][x] = 0.0f;
#pragma unroll 1
  for (int kc = 0; kc < kChunks; ++kc) {
    uint4 dv[4];
#pragma unroll
    for (int x = 0; x < 4; ++x) {
      const int a = 32 * wp + ta + 8 * x;
      dv[x] = Dtile[a * kChunks + (kc ^ (a & 7))];
    }
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const float* qk = Qb + (8 * kc + kk) * 32;
      const float4 qa = *reinterpret_cast<const float4*>(qk + (((2 * tr) ^ kk) << 2));
      const float4 qb = *reinterpret_cast<const float4*>(qk + (((2 * tr + 1) ^ kk) << 2));
      const float qq[8] = {qa.x, qa.y, qa.z, qa.w, qb.x, qb.y, qb.z, qb.w};
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        const uint32_t wv = (kk >> 1) == 0 ? dv[x].x : (kk >> 1) == 1 ? dv[x].y
                          : (kk >> 1) == 2 ? dv[x].z : dv[x].w;
        const float d = (kk & 1) ? bf16_hi(wv) : bf16_lo(wv);
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i][x] = fmaf(qq[i], d, acc[i][x]);
      }
    }
  }
  const int abase = a0 + tile * kGvAtoms + 32 * wp + ta;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int r = r0 + rb * 32 + 8 * tr + i;
    if (r >= R) continue;
    float* dst = p.qd + (int64_t)r * n;
#pragma unroll
    for (int x = 0; x < 4; ++x)
      if (abase + 8 * x < n) dst[abase + 8 * x] = acc[i][x];
  }
}

// -------------------------------------------------------------- klow_kernel
// s_lo for every (query head, token): QD[r] staged in a 32768-entry shared
// table (zero past n: every 15-bit index reads inside it, and an index >= n
// is reported once per thread after the scan), the three k_lo planes read
// four tokens at a time (16-byte loads when the planes are 16-byte
// aligned), one gather and one FMA per word.
//   kBracket = false: writes the order-preserving key of every token (one
//     16-byte store per quad; four 4-byte stores per quad cost as much as
//     the rest of the scan) and the 12-bit histogram of key bits 31..20 of
//     every head (shared-memory atomics, flushed once per segment), for the
//     radix selection of pass2_kernel and final_kernel.
//   kBracket = true: classifies every token against the head's sampled
//     bracket [lo, hi] of the k-th key (sample_kernel) as it is scored:
//     key > hi goes to the front of the selected list, lo <= key <= hi to
//     the candidates (token and key), the rest is dropped; slots come from
//     one atomic per warp and kind.  Keys are stored only with keep_keys.
constexpr int kScanThreads = 512;
// Start-up cost of one head segment in token units, from per-CTA timings at
// 256K tokens (CTAs that touched two heads against those that touched one):
// the Klow scan pays about 4 us of table staging, flush and pipeline fill
// per segment (about 11K tokens of scan), pass 2 about 5 us (histogram
// search, flush, pipeline fill: about 28K tokens).
constexpr int64_t kKlowSegCost = 11000;
constexpr int64_t kPass2SegCost = 28000;
constexpr int kKlowThreads = 1024;
// bracket mode: per-segment buffers of selected tokens and candidates
// (expected per segment at 256K tokens on 148 CTAs: about 4,500 and 2,300)
constexpr int kKlowAboveBuf = 8192;
constexpr int kKlowCandBuf = 4096;
// radix mode: two copies of the 4096-bin histogram (even and odd warps),
// which halves the collisions of the histogram atomics (a head's keys
// fall into few bins); the copies are summed when the segment flushes
constexpr int kKlowSmemHist = kTable * 4 + 2 * 4096 * 4;
constexpr int kKlowSmemBracket = kTable * 4 + (kKlowAboveBuf + 2 * kKlowCandBuf) * 4;

// QD row -> table[0..kTable), zero past n.  Eight 16-byte loads per thread
// are issued before any is stored, so the staging costs about one L2 round
// trip instead of eight.
__device__ __forceinline__ void stage_table(float* table, const float* src, int n) {
  const int nt = blockDim.x;
  if ((n & 3) == 0 && ((reinterpret_cast<uintptr_t>(src) & 15) == 0)) {
    const float4* s4 = reinterpret_cast<const float4*>(src);
    float4* d4 = reinterpret_cast<float4*>(table);
    const int n4 = n >> 2;
    for (int i0 = threadIdx.x; i0 < n4; i0 += 8 * nt) {
      float4 v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = i0 + u * nt;
        v[u] = i < n4 ? __ldg(s4 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int i = i0 + u * nt;
        if (i < n4) d4[i] = v[u];
      }
    }
  } else {
    for (int i = threadIdx.x; i < n; i += nt) table[i] = __ldg(src + i);
  }
  for (int i = n + threadIdx.x; i < kTable; i += nt) table[i] = 0.0f;
}

// kCheck: the dictionary has fewer than 32768 atoms, so an index can lie
// past it and is reported (with 32768 atoms every 15-bit index is valid).
template <bool kBracket, bool kCheck>
__global__ void __launch_bounds__(kKlowThreads, 1) klow_kernel(DecodeParams p, int vec) {
  pdl_wait();     // nothing global is touched before the previous kernel is done
  pdl_launch();
  extern __shared__ float4 smem4[];
  float* table = reinterpret_cast<float*>(smem4);
  uint32_t* sh = reinterpret_cast<uint32_t*>(table + kTable);
  uint32_t* shw = sh + ((threadIdx.x >> 5) & 1) * 4096;   // this warp's histogram copy
  // bracket mode: the segment's selected tokens and candidates are
  // collected here and reserved in the global lists once per segment
  const int cap_ab = p.klow_buf, cap_cd = p.klow_buf / 2;
  int32_t* s_ab = reinterpret_cast<int32_t*>(table + kTable);
  int32_t* s_ct = s_ab + cap_ab;
  uint32_t* s_ck = reinterpret_cast<uint32_t*>(s_ct + cap_cd);
  __shared__ uint32_t s_cnt[2], s_base[2];
  const int n = p.n, tid = threadIdx.x, lane = tid & 31;
  const int nlo = min(p.klow, kLoPlanes);
  const bool store_keys = !kBracket || p.keep_keys;
  uint32_t maxidx = 0u;
  if (kBracket && tid == 0) s_cnt[0] = s_cnt[1] = 0u;

  for_segments(p.tok_off, p.lens, p.B, p.Hq, kKlowSegCost, [&](int b, int h, int64_t t0l, int64_t t1l) {
    const int r = b * p.Hq + h, kvh = h / p.g;
    const int t0 = (int)t0l, t1 = (int)t1l;    // token indices fit 31 bits
    stage_table(table, p.qd + (int64_t)r * n, n);
    if (!kBracket)
      for (int i = tid; i < 2 * 4096; i += kKlowThreads) sh[i] = 0u;
    __syncthreads();
    const int64_t head = (int64_t)b * p.Hkv + kvh;
    const uint32_t* plane = p.k_lo + head * kLoPlanes * p.cap;
    const uint32_t* rec = p.k_full + head * p.cap * p.rs;
    uint32_t* keys = p.keys + (int64_t)r * p.L;
    sdk_select_state* st = p.st + r;
    uint32_t lo = 0u, hi = 0u;
    if (kBracket) {
      lo = __ldcg(&st->bracket_lo);
      hi = __ldcg(&st->bracket_hi);
    }
    int32_t* above_out = p.list + (int64_t)r * p.L;
    int32_t* cand_t = p.cand_t + (int64_t)r * p.L;
    uint32_t* cand_k = p.cand_key + (int64_t)r * p.L;
    // quads of 4 tokens [4q, 4q+4); the segment's edge quads are masked
    const int q0 = t0 >> 2, q1 = (t1 + 3) >> 2;
    auto load_quad = [&](int q, uint32_t (&w)[kLoPlanes][4]) {
#pragma unroll
      for (int j = 0; j < kLoPlanes; ++j) {
        if (j < nlo && q < q1) {
          if (vec) {
            const uint4 v = __ldcs(reinterpret_cast<const uint4*>(plane + j * p.cap) + q);
            w[j][0] = v.x; w[j][1] = v.y; w[j][2] = v.z; w[j][3] = v.w;
            if (4 * q < t0 || 4 * q + 4 > t1) {     // edge quad: words of other tokens
#pragma unroll
              for (int u = 0; u < 4; ++u)
                if (4 * q + u < t0 || 4 * q + u >= t1) w[j][u] = 0u;
            }
          } else {
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int t = 4 * q + u;
              w[j][u] = (t >= t0 && t < t1) ? __ldcs(plane + j * p.cap + t) : 0u;
            }
          }
        } else {
#pragma unroll
          for (int u = 0; u < 4; ++u) w[j][u] = 0u;
        }
      }
    };
    // plane lines two iterations ahead into L2 (one lane per 128-byte line)
    auto prefetch = [&](int q) {
      if (vec && q < q1 && (q & 7) == 0) {
#pragma unroll
        for (int j = 0; j < kLoPlanes; ++j)
          if (j < nlo)
            asm volatile("prefetch.global.L2 [%0];" ::"l"(
                reinterpret_cast<const uint4*>(plane + j * p.cap) + q));
      }
    };
    uint32_t wc[kLoPlanes][4], wn[kLoPlanes][4];
    load_quad(q0 + tid, wc);
    prefetch(q0 + tid + kKlowThreads);
    // every thread takes the same number of iterations (warp-wide slot
    // assignment below); quads past q1 hold no tokens
    for (int qb = q0; qb < q1; qb += kKlowThreads) {
      const int q = qb + tid;
      load_quad(q + kKlowThreads, wn);
      prefetch(q + 2 * kKlowThreads);
      uint32_t kq[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int t = 4 * q + u;
        float s = 0.0f;
#pragma unroll
        for (int j = 0; j < kLoPlanes; ++j) {
          const uint32_t idx = word_idx(wc[j][u]);
          if (kCheck) maxidx = max(maxidx, idx);
          s = fmaf(word_coef(wc[j][u]), table[idx], s);
        }
        for (int j = kLoPlanes; j < p.klow; ++j) {      // klow > 3: k_full words
          const uint32_t wj = (t >= t0 && t < t1) ? __ldg(rec + (int64_t)t * p.rs + j) : 0u;
          const uint32_t idx = word_idx(wj);
          if (kCheck) maxidx = max(maxidx, idx);
          s = fmaf(word_coef(wj), table[idx], s);
        }
        kq[u] = score_key(s);
      }
      if (store_keys) {
        // keys: one 16-byte store per whole quad (rows are 16-byte aligned)
        if (4 * q >= t0 && 4 * q + 4 <= t1) {
          *reinterpret_cast<uint4*>(keys + 4 * q) = make_uint4(kq[0], kq[1], kq[2], kq[3]);
          if (!kBracket) {
#pragma unroll
            for (int u = 0; u < 4; ++u) atomicAdd(&shw[kq[u] >> 20], 1u);
          }
        } else if (q < q1) {
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int t = 4 * q + u;
            if (t >= t0 && t < t1) {
              keys[t] = kq[u];
              if (!kBracket) atomicAdd(&shw[kq[u] >> 20], 1u);
            }
          }
        }
      }
      if (kBracket) {
        // classify; the warp's slots of each kind come from one atomic
        unsigned fa = 0u, fc = 0u;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int t = 4 * q + u;
          const bool valid = t >= t0 && t < t1;
          const bool a = valid && kq[u] > hi;
          const bool c = valid && !a && kq[u] >= lo;
          fa |= (unsigned)a << u;
          fc |= (unsigned)c << u;
        }
        const uint32_t mine = (uint32_t)__popc(fa) | ((uint32_t)__popc(fc) << 16);
        uint32_t incl = mine;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += v;
        }
        const uint32_t tot = __shfl_sync(0xffffffffu, incl, 31);
        if (tot != 0u) {
          // slots in the shared-memory buffers (one shared atomic per kind
          // and warp); past a buffer's end an entry takes a global slot
          uint32_t ba = 0u, bc = 0u;
          if (lane == 31) {
            if (tot & 0xFFFFu) ba = atomicAdd(&s_cnt[0], tot & 0xFFFFu);
            if (tot >> 16) bc = atomicAdd(&s_cnt[1], tot >> 16);
          }
          ba = __shfl_sync(0xffffffffu, ba, 31);
          bc = __shfl_sync(0xffffffffu, bc, 31);
          const uint32_t ex = incl - mine;
          uint32_t pa = ba + (ex & 0xFFFFu), pc = bc + (ex >> 16);
          // warp-uniform: do all of the warp's entries fit the buffers?
          const bool fits = ba + (tot & 0xFFFFu) <= (uint32_t)cap_ab &&
                            bc + (tot >> 16) <= (uint32_t)cap_cd;
          if (fits) {
            // common path: predicated shared-memory stores, no branches
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int t = 4 * q + u;
              const bool a = (fa >> u) & 1u, c = (fc >> u) & 1u;
              if (a) s_ab[pa] = t;
              if (c) {
                s_ct[pc] = t;
                s_ck[pc] = kq[u];
              }
              pa += a ? 1u : 0u;
              pc += c ? 1u : 0u;
            }
          } else {
            // a buffer is full: entries past its end take global slots
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int t = 4 * q + u;
              if ((fa >> u) & 1u) {
                if (pa < (uint32_t)cap_ab) {
                  s_ab[pa] = t;
                } else {
                  const uint32_t g = atomicAdd(&st->n_above, 1u);
                  if (g < (uint32_t)p.L) above_out[g] = t;
                }
                ++pa;
              }
              if ((fc >> u) & 1u) {
                if (pc < (uint32_t)cap_cd) {
                  s_ct[pc] = t;
                  s_ck[pc] = kq[u];
                } else {
                  const uint32_t g = atomicAdd(&st->n_cand, 1u);
                  if (g < (uint32_t)p.L) {
                    cand_t[g] = t;
                    cand_k[g] = kq[u];
                  }
                }
                ++pc;
              }
            }
          }
        }
      }
#pragma unroll
      for (int j = 0; j < kLoPlanes; ++j)
#pragma unroll
        for (int u = 0; u < 4; ++u) wc[j][u] = wn[j][u];
    }
    __syncthreads();
    if (!kBracket) {
      uint32_t* gh = p.hist1 + (int64_t)r * 4096;
      for (int i = tid; i < 4096; i += kKlowThreads) {
        const uint32_t c = sh[i] + sh[4096 + i];
        if (c) atomicAdd(&gh[i], c);
      }
      __syncthreads();
    } else {
      // the segment's buffered entries: one global reservation per kind
      if (tid == 0) {
        const uint32_t na = min(s_cnt[0], (uint32_t)cap_ab);
        const uint32_t nc = min(s_cnt[1], (uint32_t)cap_cd);
        s_base[0] = na ? atomicAdd(&st->n_above, na) : 0u;
        s_base[1] = nc ? atomicAdd(&st->n_cand, nc) : 0u;
      }
      __syncthreads();
      const uint32_t na = min(s_cnt[0], (uint32_t)cap_ab);
      const uint32_t nc = min(s_cnt[1], (uint32_t)cap_cd);
      for (uint32_t i = tid; i < na; i += kKlowThreads) {
        const uint32_t g = s_base[0] + i;
        if (g < (uint32_t)p.L) above_out[g] = s_ab[i];
      }
      for (uint32_t i = tid; i < nc; i += kKlowThreads) {
        const uint32_t g = s_base[1] + i;
        if (g < (uint32_t)p.L) {
          cand_t[g] = s_ct[i];
          cand_k[g] = s_ck[i];
        }
      }
      __syncthreads();
      if (tid == 0) s_cnt[0] = s_cnt[1] = 0u;
    }
  });
  if (kCheck && maxidx >= (uint32_t)n) record_error(p.hdr, SDK_ERR_DEVICE_CHECK, maxidx);
}

// ------------------------------------------------------- final selection
constexpr int kFinalStage = 12288;   // candidates staged in shared memory

// The rank-th smallest token index (1-based) among the candidates whose key
// equals T, by radix select over index digits 31..21, 20..10, 9..0 (bins
// kept in reverse so the descending search walks ascending indices).  sh:
// 2048 words of shared memory.  Sets bad when rank exceeds the ties.
__device__ uint32_t tie_cut(const uint32_t* ck, const int32_t* ct, uint32_t n_cand, uint32_t T,
                            uint32_t rank, uint32_t* s_tmp, uint32_t* sh, bool& bad) {
  const int tid = threadIdx.x;
  uint32_t prefix = 0u;
  bad = false;
  for (int ps = 0; ps < 3; ++ps) {
    const int sh_lo = ps == 0 ? 21 : (ps == 1 ? 10 : 0);
    const int wbits = ps == 2 ? 10 : 11;
    const uint32_t nb = 1u << wbits;
    for (int i = tid; i < 2048; i += blockDim.x) sh[i] = 0u;
    __syncthreads();
    for (uint32_t i = tid; i < n_cand; i += blockDim.x) {
      if (ck[i] != T) continue;
      const uint32_t t = (uint32_t)ct[i];
      const uint32_t hi = (ps == 0) ? 0u : (t >> (sh_lo + wbits));
      if (hi != prefix) continue;
      atomicAdd(&sh[2047u - ((t >> sh_lo) & (nb - 1u))], 1u);
    }
    __syncthreads();
    uint32_t bin, above, cnt;
    block_find_desc<2048>(sh, rank, s_tmp, bin, above, cnt, bad);
    if (bad) return 0u;
    prefix = (prefix << wbits) | (2047u - bin);
    rank -= above;
  }
  return prefix;
}
// The last two radix digits of one query head over its candidates, the
// exact k-th key, the tie rule (lower token index first) and the rest of the
// selected set (inputs written by pass2_kernel, read through L2).
// s_cand: 2 * kFinalStage words of shared memory; sh: 2048 words.
__device__ void final_head(const DecodeParams& p, int r, uint32_t* s_cand, uint32_t* s_tmp,
                           uint32_t* sh, uint32_t* s_cnt) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const unsigned lt = (1u << lane) - 1u;
  const int b = r / p.Hq;
  const int Nb = p.lens[b];
  const uint32_t k = (uint32_t)p.kcnt[b];
  sdk_select_state* st = p.st + r;
  const uint32_t n_cand = __ldcg(&st->n_cand);
  const uint32_t n_above = __ldcg(&st->n_above);
  if (__ldcg(&st->n_sel) != n_above || n_above >= k || n_cand == 0u || n_cand > (uint32_t)Nb) {
    if (tid == 0) record_error(p.hdr, SDK_ERR_DEVICE_CHECK, 0x20000000u | r);
    return;
  }
  const uint32_t* ck = p.cand_key + (int64_t)r * p.L;
  const int32_t* ct = p.cand_t + (int64_t)r * p.L;
  int32_t* list = p.list + (int64_t)r * p.L;
  const uint32_t k1 = k - n_above;
  // candidates in shared memory when they fit: asynchronous 16-byte copies
  // (rows are 16-byte aligned; the last copy of each array reads only the
  // remaining words) that land while the second digit is searched in hist2.
  // Otherwise the passes read global memory.
  const bool staged = n_cand <= (uint32_t)kFinalStage;
  if (staged) {
    for (uint32_t i4 = tid; 4 * i4 < n_cand; i4 += kScanThreads) {
      const unsigned bytes = 4u * min(4u, n_cand - 4 * i4);
      cp_async16_n(s_cand + 4 * i4, ck + 4 * i4, bytes);
      cp_async16_n(s_cand + kFinalStage + 4 * i4, ct + 4 * i4, bytes);
    }
    cp_async_commit();
  }

  uint32_t b2, above2, cnt2, b3, above3, cnt3;
  bool bad;
  block_find_desc<4096, true>(p.hist2 + (int64_t)r * 4096, k1, s_tmp, b2, above2, cnt2, bad);
  if (staged) {
    cp_async_wait<0>();
    __syncthreads();
    ck = s_cand;
    ct = reinterpret_cast<const int32_t*>(s_cand + kFinalStage);
  }
  if (bad) {
    if (tid == 0) record_error(p.hdr, SDK_ERR_DEVICE_CHECK, 0x21000000u | r);
    return;
  }
  const uint32_t k2 = k1 - above2;
  for (int i = tid; i < 256; i += kScanThreads) sh[i] = 0u;
  __syncthreads();
  for (uint32_t i = tid; i < n_cand; i += kScanThreads) {
    const uint32_t key = ck[i];
    if (((key >> 8) & 0xFFFu) == b2) atomicAdd(&sh[key & 0xFFu], 1u);
  }
  __syncthreads();
  block_find_desc<256>(sh, k2, s_tmp, b3, above3, cnt3, bad);
  if (bad) {
    if (tid == 0) record_error(p.hdr, SDK_ERR_DEVICE_CHECK, 0x22000000u | r);
    return;
  }
  const uint32_t b1 = ck[0] >> 20;
  const uint32_t T = (b1 << 20) | (b2 << 8) | b3;
  const uint32_t eq_take = k2 - above3;
  const uint32_t eq_total = cnt3;

  // more ties than places: the eq_take-th smallest token index among the
  // ties (tie_cut)
  uint32_t t_cut = 0xFFFFFFFFu;
  if (eq_total > eq_take) {
    t_cut = tie_cut(ck, ct, n_cand, T, eq_take, s_tmp, sh, bad);
    if (bad) {
      if (tid == 0) record_error(p.hdr, SDK_ERR_DEVICE_CHECK, 0x23000000u | r);
      return;
    }
  }

  if (tid == 0) {
    s_cnt[0] = n_above;
    s_cnt[1] = __ldcg(&st->n_comp);
  }
  __syncthreads();
  // a warp takes 4 x 32 candidates per round: one slot atomic per kind
  uint32_t cmax = 0u;
  constexpr int kU = 4;
  for (uint32_t i0 = (uint32_t)warp * 32 * kU; i0 < n_cand; i0 += kScanThreads * kU) {
    uint32_t key[kU], t[kU];
    unsigned msel[kU], mcomp[kU];
    uint32_t ns = 0u, nc = 0u;
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const uint32_t i = i0 + 32 * u + lane;
      key[u] = 0u;
      t[u] = 0u;
      bool sel = false, comp = false;
      if (i < n_cand) {
        key[u] = ck[i];
        t[u] = (uint32_t)ct[i];
        sel = key[u] > T || (key[u] == T && t[u] <= t_cut);
        comp = !sel && p.full;
      }
      msel[u] = __ballot_sync(0xffffffffu, sel);
      mcomp[u] = __ballot_sync(0xffffffffu, comp);
      ns += (uint32_t)__popc(msel[u]);
      nc += (uint32_t)__popc(mcomp[u]);
    }
    uint32_t bs = 0, bo = 0;
    if (lane == 0) {
      if (ns) bs = atomicAdd(&s_cnt[0], ns);
      if (nc) bo = atomicAdd(&s_cnt[1], nc);
    }
    bs = __shfl_sync(0xffffffffu, bs, 0);
    bo = __shfl_sync(0xffffffffu, bo, 0);
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      if (msel[u] & (1u << lane)) {
        const uint32_t pos = bs + (uint32_t)__popc(msel[u] & lt);
        if (pos < k) list[pos] = (int32_t)t[u];
        else record_error(p.hdr, SDK_ERR_DEVICE_CHECK, 0x26000000u | r);
      }
      if (mcomp[u] & (1u << lane)) {
        const uint32_t pos = bo + (uint32_t)__popc(mcomp[u] & lt);
        if (pos < (uint32_t)Nb) list[Nb - 1 - (int64_t)pos] = (int32_t)t[u];
        else record_error(p.hdr, SDK_ERR_DEVICE_CHECK, 0x27000000u | r);
        cmax = max(cmax, key[u]);
      }
      bs += (uint32_t)__popc(msel[u]);
      bo += (uint32_t)__popc(mcomp[u]);
    }
  }
  if (p.full) {
    cmax = warp_umax(cmax);
    if (lane == 0 && cmax) atomicMax(&st->max_comp, cmax);
  }
  __syncthreads();
  if (tid == 0) {
    st->kth_key = T;
    st->eq_total = eq_total;
    st->eq_taken = eq_take;
    st->n_sel = s_cnt[0];
    st->n_comp = s_cnt[1];
    if (s_cnt[0] != k) record_error(p.hdr, SDK_ERR_DEVICE_CHECK, 0x24000000u | r);
    if (p.full && s_cnt[0] + s_cnt[1] != (uint32_t)Nb)
      record_error(p.hdr, SDK_ERR_DEVICE_CHECK, 0x25000000u | r);
  }
}

// One CTA per query head runs the final selection.
__global__ void __launch_bounds__(kScanThreads) final_kernel(DecodeParams p) {
  pdl_wait();     // nothing global is touched before the previous kernel is done
  pdl_launch();
  __shared__ uint32_t s_tmp[48];
  __shared__ uint32_t sh[2048];
  __shared__ uint32_t s_cnt[2];
  extern __shared__ uint32_t s_cand[];   // 2 * kFinalStage words
  final_head(p, blockIdx.x, s_cand, s_tmp, sh, s_cnt);
}

// ------------------------------------------ sampled-bracket selection
// The exact top k per query head without a second pass over the keys:
//   sample_kernel  scores a sample of the head's tokens (sample_geom: every
//                  token when N <= 8192, else 1024 hashed runs of 8
//                  consecutive tokens) with exactly the Klow scan's
//                  arithmetic, and brackets the k-th key by two order
//                  statistics of the sample, 6 standard deviations of the
//                  sample rank on either side of the expected rank S k / N
//                  (the whole population when N <= 8192: lo = hi = the k-th
//                  key itself);
//   klow_kernel<1> selects key > hi and collects lo <= key <= hi;
//   select_kernel  finds the exact k-th key among the candidates when
//                  n_above < k <= n_above + n_cand (ties: lower token), and
//                  otherwise (the bracket missed, rare for a representative
//                  sample) re-scores the whole head and selects by radix
//                  histograms.
// The result is the same set as the radix path in every case.
constexpr int kSampleMax = 8192;
constexpr int kSampleThreads = 1024;
constexpr double kBracketSigmas = 6.0;

// The rank-th largest (1-based) of n keys.  The result lies in [lo, hi],
// first the keys' own range; every pass histograms (key - lo) >> shift
// over 2048 bins with the smallest shift that covers the range, keeps the
// bin that holds the rank-th key and narrows [lo, hi] to it, until shift
// is 0.  Scaling the bins to the range (instead of fixed key digits)
// spreads keys that share their high bits, e.g. the scores inside a
// bracket, over many bins, so the shared-memory atomics rarely collide.
// Also returns the number of keys equal to the result (cnt) and the rank
// of the result among them (rank_in_ties: rank - the number of larger
// keys).  keys: shared or global memory (written before a __syncthreads of
// this block or by an earlier kernel); hist: 2048 words of shared memory.
__device__ uint32_t rank_desc(const uint32_t* keys, int n, uint32_t rank, uint32_t* hist,
                              uint32_t* s_tmp, uint32_t& cnt, uint32_t& rank_in_ties, bool& bad) {
  const int tid = threadIdx.x, nt = blockDim.x, lane = tid & 31, warp = tid >> 5;
  uint32_t mn = 0xFFFFFFFFu, mx = 0u;
  for (int i = tid; i < n; i += nt) {
    const uint32_t key = keys[i];
    mn = min(mn, key);
    mx = max(mx, key);
  }
  mx = warp_umax(mx);
  mn = ~warp_umax(~mn);
  if (lane == 0) {
    s_tmp[warp] = mx;
    hist[warp] = mn;        // hist is free until the first pass clears it
  }
  __syncthreads();
  if (warp == 0) {
    const int nw = nt >> 5;
    uint32_t a = lane < nw ? s_tmp[lane] : 0u, c = lane < nw ? hist[lane] : 0xFFFFFFFFu;
    a = warp_umax(a);
    c = ~warp_umax(~c);
    if (lane == 0) {
      s_tmp[40] = c;
      s_tmp[41] = a;
    }
  }
  __syncthreads();
  uint32_t lo = s_tmp[40], hi = s_tmp[41];
  __syncthreads();
  cnt = 0u;
  bad = false;
  if (n <= 0 || lo > hi) {
    bad = true;
    return 0u;
  }
  while (true) {
    const uint32_t range = hi - lo;
    const int shift = range < 2048u ? 0 : (32 - __clz((int)range)) - 11;
    for (int i = tid; i < 2048; i += nt) hist[i] = 0u;
    __syncthreads();
    for (int i = tid; i < n; i += nt) {
      const uint32_t key = keys[i];
      if (key >= lo && key <= hi) atomicAdd(&hist[(key - lo) >> shift], 1u);
    }
    __syncthreads();
    uint32_t bin, above;
    block_find_desc<2048>(hist, rank, s_tmp, bin, above, cnt, bad);
    if (bad) return 0u;
    rank -= above;
    const uint32_t nlo = lo + (bin << shift);
    if (shift == 0) {
      rank_in_ties = rank;
      return nlo;
    }
    const uint64_t top = (uint64_t)nlo + ((1ull << shift) - 1ull);
    hi = top < (uint64_t)hi ? (uint32_t)top : hi;
    lo = nlo;
  }
}

// The rank-th smallest token index (1-based) among tokens 0..n-1 whose key
// equals T (tie_cut for keys indexed by token).  sh: 2048 words.
__device__ uint32_t tie_cut_tokens(const uint32_t* keys, int n, uint32_t T, uint32_t rank,
                                   uint32_t* s_tmp, uint32_t* sh, bool& bad) {
  const int tid = threadIdx.x;
  uint32_t prefix = 0u;
  bad = false;
  for (int ps = 0; ps < 3; ++ps) {
    const int sh_lo = ps == 0 ? 21 : (ps == 1 ? 10 : 0);
    const int wbits = ps == 2 ? 10 : 11;
    const uint32_t nb = 1u << wbits;
    for (int i = tid; i < 2048; i += blockDim.x) sh[i] = 0u;
    __syncthreads();
    for (int i = tid; i < n; i += blockDim.x) {
      if (keys[i] != T) continue;
      const uint32_t t = (uint32_t)i;
      const uint32_t hi = (ps == 0) ? 0u : (t >> (sh_lo + wbits));
      if (hi != prefix) continue;
      atomicAdd(&sh[2047u - ((t >> sh_lo) & (nb - 1u))], 1u);
    }
    __syncthreads();
    uint32_t bin, above, cnt;
    block_find_desc<2048>(sh, rank, s_tmp, bin, above, cnt, bad);
    if (bad) return 0u;
    prefix = (prefix << wbits) | (2047u - bin);
    rank -= above;
  }
  return prefix;
}

// s_lo of token t of a head exactly as klow_kernel computes it (the same
// words, table values and FMA order; an index >= n reads 0).
__device__ __forceinline__ float klow_score_at(const uint32_t* plane, int64_t cap,
                                               const uint32_t* rec, int rs, int t, int klow, int nlo,
                                               const float* tab, int n, bool global_tab) {
  uint32_t w[kLoPlanes];
#pragma unroll
  for (int j = 0; j < kLoPlanes; ++j) w[j] = j < nlo ? __ldg(plane + j * cap + t) : 0u;
  float s = 0.0f;
#pragma unroll
  for (int j = 0; j < kLoPlanes; ++j) {
    const uint32_t idx = word_idx(w[j]);
    const float v = global_tab ? (idx < (uint32_t)n ? __ldg(tab + idx) : 0.0f) : tab[idx];
    s = fmaf(word_coef(w[j]), v, s);
  }
  for (int j = kLoPlanes; j < klow; ++j) {
    const uint32_t wj = __ldg(rec + (int64_t)t * rs + j);
    const uint32_t idx = word_idx(wj);
    const float v = global_tab ? (idx < (uint32_t)n ? __ldg(tab + idx) : 0.0f) : tab[idx];
    s = fmaf(word_coef(wj), v, s);
  }
  return s;
}

// Geometry of the sample of an N-token head: every token when N <= 8192;
// otherwise runs of 8 consecutive tokens, one run per block of blk tokens
// (blk = 8 ceil(ceil(N / 1024) / 8)), the run of block i starting at
// i blk + 8 (lowbias32(seed ^ i) mod (len_i / 8)) with len_i = min(blk,
// N - i blk), or covering the whole block when len_i < 8.  A run of 8
// keeps every sampled plane read inside one 32-byte sector.
struct SampleGeom {
  int blk, nb, S;
};
__device__ __forceinline__ SampleGeom sample_geom(int N) {
  SampleGeom g;
  if (N <= kSampleMax) {
    g.blk = 1;
    g.nb = N;
    g.S = N;
  } else {
    g.blk = 8 * ((((N + 1023) / 1024) + 7) / 8);
    g.nb = (N + g.blk - 1) / g.blk;
    const int last = N - (g.nb - 1) * g.blk;
    g.S = 8 * (g.nb - 1) + min(8, last);
  }
  return g;
}
// Token of sample i (0 <= i < S).
__device__ __forceinline__ int sample_token(const SampleGeom& g, int N, uint32_t seed, int i) {
  if (g.blk == 1) return i;
  const int run = i >> 3, pos = i & 7;
  const int len = min(g.blk, N - run * g.blk);
  const int off = len < 8 ? 0 : 8 * (int)(lowbias32(seed ^ (uint32_t)run) % (uint32_t)(len / 8));
  return run * g.blk + off + pos;
}

// One CTA per query head: the sample, its keys and the bracket [lo, hi].
// QD of the head is staged in shared memory as in the Klow scan (the same
// table values, so a sampled token's key equals its scan key).
constexpr int kSampleSmem = kTable * 4;
__global__ void __launch_bounds__(kSampleThreads, 1) sample_kernel(DecodeParams p) {
  pdl_wait();
  pdl_launch();
  extern __shared__ float4 smem4[];
  float* table = reinterpret_cast<float*>(smem4);
  __shared__ uint32_t s_key[kSampleMax];
  __shared__ uint32_t s_hist[2048];
  __shared__ uint32_t s_tmp[48];
  const int r = blockIdx.x, tid = threadIdx.x;
  const int b = r / p.Hq, h = r % p.Hq, kvh = h / p.g;
  const int N = p.lens[b], k = p.kcnt[b];
  const SampleGeom gm = sample_geom(N);
  const int S = gm.S;
  const int64_t head = (int64_t)b * p.Hkv + kvh;
  const uint32_t* plane = p.k_lo + head * kLoPlanes * p.cap;
  const uint32_t* rec = p.k_full + head * p.cap * p.rs;
  const uint32_t seed = lowbias32(0x9E3779B9u * (uint32_t)(head + 1));
  const int nlo = min(p.klow, kLoPlanes);
  // up to 8 samples per thread; their plane words are requested before the
  // table is staged, so the two round trips overlap
  constexpr int kPer = kSampleMax / kSampleThreads;
  int tt[kPer];
  uint32_t wv[kPer][kLoPlanes];
#pragma unroll
  for (int u = 0; u < kPer; ++u) {
    const int i = tid + u * kSampleThreads;
    tt[u] = i < S ? sample_token(gm, N, seed, i) : -1;
#pragma unroll
    for (int j = 0; j < kLoPlanes; ++j)
      wv[u][j] = (tt[u] >= 0 && j < nlo) ? __ldg(plane + j * p.cap + tt[u]) : 0u;
  }
  stage_table(table, p.qd + (int64_t)r * p.n, p.n);
  __syncthreads();
#pragma unroll
  for (int u = 0; u < kPer; ++u) {
    if (tt[u] < 0) continue;
    float s = 0.0f;
#pragma unroll
    for (int j = 0; j < kLoPlanes; ++j) s = fmaf(word_coef(wv[u][j]), table[word_idx(wv[u][j])], s);
    for (int j = kLoPlanes; j < p.klow; ++j) {
      const uint32_t wj = __ldg(rec + (int64_t)tt[u] * p.rs + j);
      s = fmaf(word_coef(wj), table[word_idx(wj)], s);
    }
    s_key[tid + u * kSampleThreads] = score_key(s);
  }
  __syncthreads();
  // sample ranks of the bracket (1-based, descending); 0 = no upper end
  // (nothing is selected directly), S + 1 = no lower end (every token not
  // above hi is a candidate)
  int rhi, rlo;
  if (S == N) {
    rhi = rlo = k;
  } else if (k >= N) {
    rhi = 0;
    rlo = S + 1;
  } else {
    const double pp = (double)k / (double)N;
    const double mu = (double)S * pp, sg = sqrt((double)S * pp * (1.0 - pp));
    const double a = floor(mu - kBracketSigmas * sg), c = ceil(mu + kBracketSigmas * sg);
    rhi = a < 1.0 ? 0 : (int)a;
    rlo = c > (double)S ? S + 1 : (int)c;
  }
  uint32_t hi = 0xFFFFFFFFu, lo = 0u, cnt, rit;
  bool bad = false;
  if (rhi >= 1) hi = rank_desc(s_key, S, (uint32_t)rhi, s_hist, s_tmp, cnt, rit, bad);
  if (!bad && rlo <= S) lo = rank_desc(s_key, S, (uint32_t)rlo, s_hist, s_tmp, cnt, rit, bad);
  if (tid == 0) {
    if (bad) {           // cannot happen for 1 <= rank <= S; select_kernel re-scans
      hi = 0u;
      lo = 0xFFFFFFFFu;
      record_error(p.hdr, SDK_ERR_DEVICE_CHECK, 0x28000000u | r);
    }
    sdk_select_state* st = p.st + r;
    st->bracket_lo = lo;
    st->bracket_hi = hi;
    st->select_path = 1u;
  }
}

constexpr int kSelThreads = 1024;
constexpr int kSelStage = kTable / 2;      // staged candidates: keys + tokens = 128 KB
constexpr int kSelSmem = kTable * 4;       // the same bytes hold the fallback's QD table

// Appends the tokens selected by (key > T, or key == T and token <= t_cut)
// among n entries (key_at(i), tok_at(i)) to list at slots from s_cnt[0].
template <class KeyAt, class TokAt>
__device__ __forceinline__ void append_selected(int n, uint32_t T, uint32_t t_cut, KeyAt key_at,
                                                TokAt tok_at, int32_t* list, uint32_t k,
                                                uint32_t* s_cnt, WsHeader* hdr, int r) {
  const int tid = threadIdx.x, lane = tid & 31;
  const unsigned lt = (1u << lane) - 1u;
  for (int i0 = tid - lane; i0 < n; i0 += kSelThreads) {
    const int i = i0 + lane;
    bool sel = false;
    uint32_t t = 0u;
    if (i < n) {
      const uint32_t key = key_at(i);
      t = tok_at(i);
      sel = key > T || (key == T && t <= t_cut);
    }
    const unsigned m = __ballot_sync(0xffffffffu, sel);
    uint32_t base = 0u;
    if (lane == 0 && m) base = atomicAdd(&s_cnt[0], (uint32_t)__popc(m));
    base = __shfl_sync(0xffffffffu, base, 0);
    if (sel) {
      const uint32_t pos = base + (uint32_t)__popc(m & lt);
      if (pos < k) list[pos] = (int32_t)t;
      else record_error(hdr, SDK_ERR_DEVICE_CHECK, 0x26000000u | r);
    }
  }
}

// One CTA per query head: the rest of the selected set (bracket path), or
// the whole selection by an exact re-scan when the bracket missed.
__global__ void __launch_bounds__(kSelThreads, 1) select_kernel(DecodeParams p) {
  pdl_wait();
  pdl_launch();
  extern __shared__ float4 smem4[];
  __shared__ uint32_t sh[2048];
  __shared__ uint32_t s_tmp[48];
  __shared__ uint32_t s_cnt[2];
  const int r = blockIdx.x, tid = threadIdx.x;
  const int b = r / p.Hq, h = r % p.Hq, kvh = h / p.g;
  const int N = p.lens[b];
  const uint32_t k = (uint32_t)p.kcnt[b];
  sdk_select_state* st = p.st + r;
  const uint32_t A = __ldcg(&st->n_above), C = __ldcg(&st->n_cand);
  int32_t* list = p.list + (int64_t)r * p.L;
  uint32_t T = 0u, eq_total = 0u, eq_take = 0u, t_cut = 0xFFFFFFFFu;
  bool bad = false;
  const bool hit = A < k && (uint64_t)A + C >= k && A + C <= (uint32_t)N;
  if (hit) {
    // the (k - A)-th largest candidate, staged in shared memory when the
    // candidates fit (otherwise read through L2)
    const uint32_t* ck = p.cand_key + (int64_t)r * p.L;
    const int32_t* ct = p.cand_t + (int64_t)r * p.L;
    if (C <= (uint32_t)kSelStage) {
      // 16-byte asynchronous copies, all of a thread's in flight at once
      // (rows are 16-byte aligned; the last copy reads only what is left)
      uint32_t* s_ck = reinterpret_cast<uint32_t*>(smem4);
      int32_t* s_ct = reinterpret_cast<int32_t*>(s_ck + kSelStage);
      for (uint32_t i4 = tid; 4 * i4 < C; i4 += kSelThreads) {
        const unsigned bytes = 4u * min(4u, C - 4 * i4);
        cp_async16_n(s_ck + 4 * i4, ck + 4 * i4, bytes);
        cp_async16_n(s_ct + 4 * i4, ct + 4 * i4, bytes);
      }
      cp_async_commit();
      cp_async_wait<0>();
      __syncthreads();
      ck = s_ck;
      ct = s_ct;
    }
    const uint32_t k1 = k - A;
    T = rank_desc(ck, (int)C, k1, sh, s_tmp, eq_total, eq_take, bad);
    if (!bad && eq_total > eq_take) t_cut = tie_cut(ck, ct, C, T, eq_take, s_tmp, sh, bad);
    if (bad) {
      if (tid == 0) record_error(p.hdr, SDK_ERR_DEVICE_CHECK, 0x29000000u | r);
      return;
    }
    if (tid == 0) s_cnt[0] = A;
    __syncthreads();
    append_selected((int)C, T, t_cut, [&](int i) { return ck[i]; },
                    [&](int i) { return (uint32_t)ct[i]; }, list, k, s_cnt, p.hdr, r);
  } else {
    // exact re-scan: every token's key into `keys`, then the radix select
    float* table = reinterpret_cast<float*>(smem4);
    stage_table(table, p.qd + (int64_t)r * p.n, p.n);
    __syncthreads();
    const int64_t head = (int64_t)b * p.Hkv + kvh;
    const uint32_t* plane = p.k_lo + head * kLoPlanes * p.cap;
    const uint32_t* rec = p.k_full + head * p.cap * p.rs;
    uint32_t* keys = p.keys + (int64_t)r * p.L;
    const int nlo = min(p.klow, kLoPlanes);
    for (int t = tid; t < N; t += kSelThreads)
      keys[t] = score_key(klow_score_at(plane, p.cap, rec, p.rs, t, p.klow, nlo, table, p.n, false));
    __syncthreads();
    T = rank_desc(keys, N, k, sh, s_tmp, eq_total, eq_take, bad);
    if (!bad && eq_total > eq_take) t_cut = tie_cut_tokens(keys, N, T, eq_take, s_tmp, sh, bad);
    if (bad) {
      if (tid == 0) record_error(p.hdr, SDK_ERR_DEVICE_CHECK, 0x2A000000u | r);
      return;
    }
    if (tid == 0) s_cnt[0] = 0u;
    __syncthreads();
    append_selected(N, T, t_cut, [&](int i) { return keys[i]; },
                    [&](int i) { return (uint32_t)i; }, list, k, s_cnt, p.hdr, r);
  }
  __syncthreads();
  if (tid == 0) {
    st->kth_key = T;
    st->eq_total = eq_total;
    st->eq_taken = eq_take;
    st->n_sel = s_cnt[0];
    st->select_path = hit ? 1u : 2u;
    if (s_cnt[0] != k) record_error(p.hdr, SDK_ERR_DEVICE_CHECK, 0x24000000u | r);
  }
}

// ------------------------------------------- context-sharded final stages
// A rank holds a contiguous token range of every sequence (ranks in token
// order).  After klow the ranks sum hist1, so pass2 finds the global bucket
// of the k-th key; the last two digits and the ties follow here in three
// stages, with the ranks combining, between them, the regions that the
// unsharded path has finished with:
//   stage 3 writes hist3 [R][256] (third digit over the local candidates)
//           at the start of hist1; the ranks sum it;
//   stage 4 writes the local tie count [R] at the start of hist2; the ranks
//           gather it into ties[world][R];
//   stage 5 selects the local candidates above the k-th key and the rank's
//           share of the ties (ties are taken in global token order, i.e.
//           lower ranks first), completing the local selected list.
// State carried in sdk_select_state: kth_key (b1 << 20 from pass2, then
// with b2, then the key T), eq_taken (k2, then the ties to take over all
// ranks), eq_total (all ties), n_sel (the local selected count).
__device__ __forceinline__ bool shard_head_ok(const DecodeParams& p, int r,
                                              const sdk_select_state* st) {
  const uint32_t k = (uint32_t)p.kcnt[r / p.Hq];
  const uint32_t n_above = __ldcg(&st->n_above);
  return n_above < k && __ldcg(&st->n_cand) <= (uint32_t)p.lens[r / p.Hq];
}

__global__ void __launch_bounds__(kScanThreads) shard_digit3_kernel(DecodeParams p) {
  __shared__ uint32_t s_tmp[48];
  __shared__ uint32_t sh[256];
  const int r = blockIdx.x, tid = threadIdx.x;
  sdk_select_state* st = p.st + r;
  if (!shard_head_ok(p, r, st)) {
    if (tid == 0) record_error(p.hdr, SDK_ERR_DEVICE_CHECK, 0x28000000u | r);
    return;
  }
  const uint32_t k1 = (uint32_t)p.kcnt[r / p.Hq] - __ldcg(&st->n_above);
  uint32_t b2, above2, cnt2;
  bool bad;
  block_find_desc<4096, true>(p.hist2 + (int64_t)r * 4096, k1, s_tmp, b2, above2, cnt2, bad);
  if (bad) {
    if (tid == 0) record_error(p.hdr, SDK_ERR_DEVICE_CHECK, 0x29000000u | r);
    return;
  }
  for (int i = tid; i < 256; i += kScanThreads) sh[i] = 0u;
  __syncthreads();
  const uint32_t n_cand = __ldcg(&st->n_cand);
  const uint32_t* ck = p.cand_key + (int64_t)r * p.L;
  for (uint32_t i = tid; i < n_cand; i += kScanThreads) {
    const uint32_t key = __ldcg(ck + i);
    if (((key >> 8) & 0xFFFu) == b2) atomicAdd(&sh[key & 0xFFu], 1u);
  }
  __syncthreads();
  for (int i = tid; i < 256; i += kScanThreads) p.hist1[(int64_t)r * 256 + i] = sh[i];
  if (tid == 0) {
    st->kth_key = __ldcg(&st->kth_key) | (b2 << 8);
    st->eq_taken = k1 - above2;   // k2
  }
}

__global__ void __launch_bounds__(kScanThreads) shard_ties_kernel(DecodeParams p) {
  __shared__ uint32_t s_tmp[48];
  __shared__ uint32_t s_cnt;
  const int r = blockIdx.x, tid = threadIdx.x;
  sdk_select_state* st = p.st + r;
  if (!shard_head_ok(p, r, st)) return;   // reported by the previous stage
  const uint32_t k2 = __ldcg(&st->eq_taken);
  uint32_t b3, above3, cnt3;
  bool bad;
  block_find_desc<256, true>(p.hist1 + (int64_t)r * 256, k2, s_tmp, b3, above3, cnt3, bad);
  if (bad) {
    if (tid == 0) record_error(p.hdr, SDK_ERR_DEVICE_CHECK, 0x2A000000u | r);
    return;
  }
  const uint32_t T = __ldcg(&st->kth_key) | b3;
  if (tid == 0) s_cnt = 0u;
  __syncthreads();
  const uint32_t n_cand = __ldcg(&st->n_cand);
  const uint32_t* ck = p.cand_key + (int64_t)r * p.L;
  uint32_t c = 0u;
  for (uint32_t i = tid; i < n_cand; i += kScanThreads) c += __ldcg(ck + i) == T ? 1u : 0u;
  c = __reduce_add_sync(0xffffffffu, c);
  if ((tid & 31) == 0 && c) atomicAdd(&s_cnt, c);
  __syncthreads();
  if (tid == 0) {
    p.hist2[r] = s_cnt;          // the local ties, gathered over the ranks
    st->kth_key = T;
    st->eq_taken = k2 - above3;  // ties to take over all ranks
    st->eq_total = cnt3;
  }
}

// ties: device, uint32 [world][R], every rank's local tie count
__global__ void __launch_bounds__(kScanThreads) shard_select_kernel(DecodeParams p,
                                                                    const uint32_t* ties,
                                                                    int rank_id) {
  __shared__ uint32_t s_tmp[48];
  __shared__ uint32_t sh[2048];
  __shared__ uint32_t s_cnt;
  const int r = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const unsigned lt = (1u << lane) - 1u;
  sdk_select_state* st = p.st + r;
  if (!shard_head_ok(p, r, st)) return;
  const int b = r / p.Hq;
  const int Nb = p.lens[b];
  const uint32_t T = __ldcg(&st->kth_key);
  const uint32_t take_all = __ldcg(&st->eq_taken);
  uint32_t before = 0u;
  for (int w = 0; w < rank_id; ++w) before += __ldcg(ties + (int64_t)w * p.R + r);
  const uint32_t mine = __ldcg(ties + (int64_t)rank_id * p.R + r);
  const uint32_t quota = take_all > before ? min(take_all - before, mine) : 0u;
  const uint32_t n_cand = __ldcg(&st->n_cand);
  const uint32_t* ck = p.cand_key + (int64_t)r * p.L;
  const int32_t* ct = p.cand_t + (int64_t)r * p.L;
  int32_t* list = p.list + (int64_t)r * p.L;
  // ties to take here: none, all, or the quota smallest indices
  bool take_ties = quota > 0u;
  uint32_t t_cut = 0xFFFFFFFFu;
  if (take_ties && quota < mine) {
    bool bad;
    t_cut = tie_cut(ck, ct, n_cand, T, quota, s_tmp, sh, bad);
    if (bad) {
      if (tid == 0) record_error(p.hdr, SDK_ERR_DEVICE_CHECK, 0x2B000000u | r);
      return;
    }
  }
  if (tid == 0) s_cnt = __ldcg(&st->n_sel);   // the local tokens above the bucket
  __syncthreads();
  for (uint32_t i0 = (uint32_t)warp * 32; i0 < n_cand; i0 += kScanThreads) {
    const uint32_t i = i0 + lane;
    bool sel = false;
    uint32_t t = 0u;
    if (i < n_cand) {
      const uint32_t key = __ldcg(ck + i);
      t = (uint32_t)__ldcg(ct + i);
      sel = key > T || (key == T && take_ties && t <= t_cut);
    }
    const unsigned msel = __ballot_sync(0xffffffffu, sel);
    uint32_t bs = 0;
    if (lane == 0 && msel) bs = atomicAdd(&s_cnt, (uint32_t)__popc(msel));
    bs = __shfl_sync(0xffffffffu, bs, 0) + __popc(msel & lt);
    if (sel) {
      if (bs < (uint32_t)Nb) list[bs] = (int32_t)t;
      else record_error(p.hdr, SDK_ERR_DEVICE_CHECK, 0x2C000000u | r);
    }
  }
  __syncthreads();
  if (tid == 0) st->n_sel = s_cnt;
}

// ------------------------------------------------------------- pass2_kernel
// Tokens above the bucket of the k-th key are selected, tokens inside it
// become candidates (with a histogram of key bits 19..8), the others go to
// the complement (full-softmax flag only).  A warp takes 512 tokens per
// step: each lane takes 16 consecutive keys (four 16-byte copies streamed
// through a per-lane shared-memory ring one step ahead), counts its tokens
// of each kind, and a warp scan gives every lane its output slots behind
// one atomic per warp and kind.  The steps are chains of dependent warp
// operations, so the CTA runs 32 warps with a short ring (measured faster
// than 16 or 24 warps with deeper rings).  Candidates and their histogram
// go through shared memory (flushed once per segment; slots past the
// buffer go straight to global memory).  The few tokens before the first
// 16-byte boundary of a segment and after its last one take a scalar path.
constexpr int kCandBuf = 2048;
constexpr int kP2Threads = 1024;
constexpr int kP2Stages = 2;                            // key ring depth per lane
constexpr int kP2RingOff = 2 * kCandBuf + 4096;         // in words
constexpr int kPass2Smem = (kP2RingOff + kP2Stages * (kP2Threads / 32) * 128 * 4) * 4;

__device__ __forceinline__ uint32_t warp_excl_scan(uint32_t v, uint32_t& total) {
  const int lane = threadIdx.x & 31;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  total = __shfl_sync(0xffffffffu, x, 31);
  return x - v;
}

__global__ void __launch_bounds__(kP2Threads, 1) pass2_kernel(DecodeParams p) {
  pdl_wait();     // nothing global is touched before the previous kernel is done
  pdl_launch();
  __shared__ uint32_t s_tmp[48];
  __shared__ uint32_t s_ncand, s_cbase;
  extern __shared__ uint32_t s_dyn[];   // kPass2Smem bytes
  int32_t* s_ct = reinterpret_cast<int32_t*>(s_dyn);
  uint32_t* s_ck = reinterpret_cast<uint32_t*>(s_ct + kCandBuf);
  uint32_t* s_h2 = s_ck + kCandBuf;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int kWarps = kP2Threads / 32;

  for_segments(p.tok_off, p.lens, p.B, p.Hq, kPass2SegCost, [&](int b, int h, int64_t t0l, int64_t t1l) {
    const int r = b * p.Hq + h;
    const int Nb = p.lens[b];
    const int t0 = (int)t0l, t1 = (int)t1l;
    sdk_select_state* st = p.st + r;
    uint32_t b1, above1, cnt1;
    bool bad;
    for (int i = tid; i < 4096; i += kP2Threads) s_h2[i] = 0u;
    if (tid == 0) s_ncand = 0u;
    block_find_desc<4096>(p.hist1 + (int64_t)r * 4096, (uint32_t)p.kcnt[b], s_tmp, b1, above1,
                          cnt1, bad);   // ends with a barrier
    if (bad) {
      if (tid == 0) record_error(p.hdr, SDK_ERR_DEVICE_CHECK, 0x10000000u | r);
      return;
    }
    if (t0 == 0 && tid == 0) {
      st->n_above = above1;
      st->kth_key = b1 << 20;   // the first digit (the final stage completes the key)
    }
    const uint32_t kLo = b1 << 20, kHi = kLo | 0xFFFFFu;   // the k-th key's bucket
    const uint32_t* keys = p.keys + (int64_t)r * p.L;
    int32_t* list = p.list + (int64_t)r * p.L;
    int32_t* ct = p.cand_t + (int64_t)r * p.L;
    uint32_t* ck = p.cand_key + (int64_t)r * p.L;
    const bool full = p.full != 0;
    uint32_t cmax = 0u;

    // one warp-wide step over up to 16 tokens per lane: tt(j) gives the
    // token of key j of this lane, kk[j] its key (valid when ok(j))
    auto step = [&](const uint32_t (&kk)[16], auto tt, auto ok) {
      uint32_t ns = 0u, nc = 0u, no = 0u;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        if (!ok(j)) continue;
        const uint32_t d1 = kk[j] >> 20;
        ns += d1 > b1 ? 1u : 0u;
        nc += d1 == b1 ? 1u : 0u;
        no += d1 < b1 ? 1u : 0u;
      }
      uint32_t tot;
      uint32_t pos = warp_excl_scan(ns, tot);
      if (tot) {
        uint32_t base = 0u;
        if (lane == 0) base = atomicAdd(&st->n_sel, tot);
        pos += __shfl_sync(0xffffffffu, base, 0);
#pragma unroll
        for (int j = 0; j < 16; ++j)
          if (ok(j) && (kk[j] >> 20) > b1) {
            if (pos < (uint32_t)Nb) list[pos] = tt(j);
            ++pos;
          }
      }
      if (__any_sync(0xffffffffu, nc != 0u)) {
        uint32_t cpos = warp_excl_scan(nc, tot);
        uint32_t base = 0u;
        if (lane == 0) base = atomicAdd(&s_ncand, tot);
        cpos += __shfl_sync(0xffffffffu, base, 0);
#pragma unroll
        for (int j = 0; j < 16; ++j)
          if (ok(j) && (kk[j] >> 20) == b1) {
            if (cpos < (uint32_t)kCandBuf) {
              s_ct[cpos] = tt(j);
              s_ck[cpos] = kk[j];
            } else {
              const uint32_t g = atomicAdd(&st->n_cand, 1u);   // rare overflow
              if (g < (uint32_t)Nb) {
                ct[g] = tt(j);
                ck[g] = kk[j];
              }
            }
            atomicAdd(&s_h2[(kk[j] >> 8) & 0xFFFu], 1u);
            ++cpos;
          }
      }
      if (full && __any_sync(0xffffffffu, no != 0u)) {
        uint32_t opos = warp_excl_scan(no, tot);
        uint32_t base = 0u;
        if (lane == 0) base = atomicAdd(&st->n_comp, tot);
        opos += __shfl_sync(0xffffffffu, base, 0);
#pragma unroll
        for (int j = 0; j < 16; ++j)
          if (ok(j) && (kk[j] >> 20) < b1) {
            if (opos < (uint32_t)Nb) list[Nb - 1 - (int)opos] = tt(j);
            cmax = max(cmax, kk[j]);
            ++opos;
          }
      }
    };

    // scalar edges: tokens before the first 16-byte boundary and after the
    // last one (at most 3 + 3), taken by warp 0
    const int lead = (int)((4u - (uint32_t)((reinterpret_cast<uintptr_t>(keys + t0) >> 2) & 3u)) & 3u);
    const int ta = min(t1, t0 + lead);
    const int tb = ta + ((t1 - ta) & ~3);
    if (warp == 0) {
      uint32_t kk[16];
      const int ne = (ta - t0) + (t1 - tb);
      auto edge_t = [&](int j) { return j < ta - t0 ? t0 + j : tb + (j - (ta - t0)); };
#pragma unroll
      for (int j = 0; j < 16; ++j) kk[j] = 0u;
      if (lane == 0) {
#pragma unroll
        for (int j = 0; j < 8; ++j)
          if (j < ne) kk[j] = keys[edge_t(j)];
      }
      step(kk, edge_t, [&](int j) { return lane == 0 && j < ne; });
    }
    // body: whole quads [ta, tb) (keys + ta is 16-byte aligned), 512
    // tokens per warp step; quad q holds tokens ta + 4q .. ta + 4q + 3.  Each
    // lane streams its four quads per step through a kP2Stages-deep ring in
    // shared memory (cp.async), so kP2Stages - 1 steps are in flight.
    const int q1 = (tb - ta) >> 2;
    const uint4* kq = reinterpret_cast<const uint4*>(keys + ta);
    uint4* ring = reinterpret_cast<uint4*>(s_dyn + kP2RingOff) + warp * (kP2Stages * 128);
    auto issue = [&](int qb, int slot) {
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const int q = qb + lane + 32 * v;
        cp_async16(ring + slot * 128 + 32 * v + lane, q < q1 ? kq + q : kq, q < q1);
      }
      cp_async_commit();
    };
    constexpr int kStride = kWarps * 128;
    const int qfirst = warp * 128;
    // selected tokens of the previous step, written once its slots are known
    uint32_t pend_msel = 0u, pend_pos = 0u, pend_rsv = 0u;
    int pend_qb = 0;
    auto write_sel = [&]() {
      const uint32_t base = __shfl_sync(0xffffffffu, pend_rsv, 0);
      uint32_t pos = base + pend_pos;
      for (uint32_t m = pend_msel; m; m &= m - 1u, ++pos) {
        const int j = __ffs(m) - 1;
        if (pos < (uint32_t)Nb) list[pos] = ta + 4 * (pend_qb + lane + 32 * (j >> 2)) + (j & 3);
      }
    };
#pragma unroll
    for (int s2 = 0; s2 < kP2Stages - 1; ++s2) issue(qfirst + s2 * kStride, s2);
    int slot = 0;
    for (int qb = qfirst; qb < q1; qb += kStride) {
      issue(qb + (kP2Stages - 1) * kStride, (slot + kP2Stages - 1) % kP2Stages);
      cp_async_wait<kP2Stages - 1>();
      // classify the lane's 16 keys into bit masks (bit j = key j), then
      // walk only the set bits
      const uint4* rs = ring + slot * 128 + lane;
      uint32_t msel = 0u, mcand = 0u, mval = 0u;
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const uint4 x = rs[32 * v];
        const uint32_t kv[4] = {x.x, x.y, x.z, x.w};
        if (qb + lane + 32 * v < q1) mval |= 0xFu << (4 * v);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          if (kv[u] > kHi) msel |= 1u << (4 * v + u);
          if (kv[u] >= kLo) mcand |= 1u << (4 * v + u);
        }
      }
      msel &= mval;
      mcand &= mval & ~msel;
      auto tok = [&](int j) { return ta + 4 * (qb + lane + 32 * (j >> 2)) + (j & 3); };
      auto key_at = [&](int j) {
        const uint4 x = rs[32 * (j >> 2)];
        const int u = j & 3;
        return u == 0 ? x.x : u == 1 ? x.y : u == 2 ? x.z : x.w;
      };
      uint32_t tot;
      // the slots of this step's selected tokens are reserved now and
      // written one step later, so the atomic's round trip overlaps a step
      const uint32_t pos = warp_excl_scan((uint32_t)__popc(msel), tot);
      const uint32_t rsv = (lane == 0 && tot) ? atomicAdd(&st->n_sel, tot) : 0u;
      write_sel();
      pend_msel = msel;
      pend_pos = pos;
      pend_rsv = rsv;
      pend_qb = qb;
      if (__any_sync(0xffffffffu, mcand != 0u)) {
        uint32_t cpos = warp_excl_scan((uint32_t)__popc(mcand), tot);
        uint32_t base = 0u;
        if (lane == 0) base = atomicAdd(&s_ncand, tot);
        cpos += __shfl_sync(0xffffffffu, base, 0);
        for (uint32_t m = mcand; m; m &= m - 1u, ++cpos) {
          const int j = __ffs(m) - 1;
          const uint32_t key = key_at(j);
          if (cpos < (uint32_t)kCandBuf) {
            s_ct[cpos] = tok(j);
            s_ck[cpos] = key;
          } else {
            const uint32_t g = atomicAdd(&st->n_cand, 1u);   // rare overflow
            if (g < (uint32_t)Nb) {
              ct[g] = tok(j);
              ck[g] = key;
            }
          }
          atomicAdd(&s_h2[(key >> 8) & 0xFFFu], 1u);
        }
      }
      if (full) {
        const uint32_t mo = mval & ~msel & ~mcand;
        uint32_t opos = warp_excl_scan((uint32_t)__popc(mo), tot);
        if (tot) {
          uint32_t base = 0u;
          if (lane == 0) base = atomicAdd(&st->n_comp, tot);
          opos += __shfl_sync(0xffffffffu, base, 0);
          for (uint32_t m = mo; m; m &= m - 1u, ++opos) {
            const int j = __ffs(m) - 1;
            if (opos < (uint32_t)Nb) list[Nb - 1 - (int)opos] = tok(j);
            cmax = max(cmax, key_at(j));
          }
        }
      }
      slot = slot + 1 == kP2Stages ? 0 : slot + 1;
    }
    write_sel();
    cp_async_wait<0>();   // drain the copies issued past the end
    __syncthreads();
    // flush the candidates and the histogram of this segment
    if (tid == 0) {
      s_ncand = min(s_ncand, (uint32_t)kCandBuf);
      s_cbase = s_ncand ? atomicAdd(&st->n_cand, s_ncand) : 0u;
    }
    __syncthreads();
    const uint32_t ncand = s_ncand, cbase = s_cbase;
    for (uint32_t i = tid; i < ncand; i += kP2Threads)
      if (cbase + i < (uint32_t)Nb) {
        ct[cbase + i] = s_ct[i];
        ck[cbase + i] = s_ck[i];
      }
    uint32_t* h2 = p.hist2 + (int64_t)r * 4096;
    for (int i = tid; i < 4096; i += kP2Threads)
      if (s_h2[i]) atomicAdd(&h2[i], s_h2[i]);
    if (full) {
      cmax = warp_umax(cmax);
      if (lane == 0 && cmax) atomicMax(&st->max_comp, cmax);
    }
    __syncthreads();
  });
}

// ------------------------------------------------------------ attend_kernel
// Khigh rescore, softmax and value scatter of one query head, fused.  One
// cluster of C CTAs per head; CTA `rank` owns the slice
// [k*rank/C, k*(rank+1)/C) of the head's selected entries list[0..k-1] and,
// with the full-softmax flag, a slice of the complement entries
// list[k..N-1] (logit scale * s_lo).  One thread per entry: it loads the
// whole 64-byte record (four 16-byte loads) and walks its 16 words.
//   phase 1  QD[r] is staged in a 32768-entry shared table (zero past n, so
//            every 15-bit index reads inside it; with n < 32768 an index >= n
//            adds 0 and is reported after the loop).  s_i = scale *
//            sum_{j<khigh} c_tj QD[idx_tj] for the own selected entries,
//            written to sel_score, with a running maximum and a running
//            sum of exp(s - running max) per thread (online softmax).  The
//            cluster's maximum m comes through distributed shared memory
//            (with the flag, also the largest complement logit), then z.
//   phase 2  the table becomes the per-atom weight tile: w[idx^V] += p c^V
//            with p = exp(logit - m) / z, in 2^-20 fixed point (native int32
//            shared-memory atomics: exact and order-independent).  Since
//            sum p = 1, a bin can leave the int32 range only if the CTA's
//            sum of |p c| reaches 2^10; a CTA that sees that re-runs the
//            phase with fp32 atomics.
//   phase 3  each CTA sums its slice of the atoms over the cluster's tiles
//            and writes the normalised w[r].
constexpr int kAttThreads = 768;
constexpr int kAttThreadsReg = 640;          // records in registers: up to 96 per thread
// shared memory: the QD / weight table, then a two-slot record ring
constexpr int kAttSmem = kTable * 4 + 2 * kAttThreads * 64;
constexpr int kAttSmemReg = kTable * 4;      // records in registers: the table only
constexpr float kFixScale = 1048576.0f;       // 2^20
constexpr float kFixInv = 1.0f / 1048576.0f;

// L2 policies: keep a line (evict last) / let it go first
__device__ __forceinline__ uint64_t l2_evict_last() {
  uint64_t pol;
  asm("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}
__device__ __forceinline__ uint64_t l2_evict_first() {
  uint64_t pol;
  asm("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// Calls f(i, t, w, x) for every entry i in [e0, e1) of `list` owned by this
// thread (i = e0 + tid + j*T); w holds the 16 words of token t's record and
// x = pay(i, t), a per-entry value whose load is issued together with the
// record's copy.  Entries naming a token outside [0, Nb) are reported and
// skipped.  Records stream through a two-slot ring per thread in shared
// memory (cp.async; the four 16-byte chunks of a slot are XOR-swizzled by
// thread so the reads are free of bank conflicts): entries i + T and i + 2T
// are in flight while i is used and the record of i + 3T is prefetched into
// L2.  The list entries themselves are loaded six iterations ahead, so no
// iteration waits on a list load.  rs4: 16-byte units between consecutive
// tokens' records (4, or 8 in the interleaved layout).  kLine: the copies
// and the prefetch bring the record's whole 128-byte line into L2 (in the
// interleaved layout the key pass thereby fetches the value record the
// value pass reads next); otherwise exactly the record's 64 bytes, since
// records sit at random token positions.
template <bool kLine, class Pay, class F>
__device__ __forceinline__ void for_records(const int32_t* list, int e0, int e1, const uint4* rec,
                                            int rs4, int Nb, WsHeader* hdr, uint32_t tag,
                                            uint4* ring, Pay pay, F f) {
  constexpr int T = kAttThreads;
  const int tid = threadIdx.x;
  const int sw = (tid >> 1) & 3;
  auto list_at = [&](int i) -> int { return i < e1 ? __ldg(list + i) : -1; };
  auto ok = [&](int t) { return (unsigned)t < (unsigned)Nb; };
  // interleaved records: the key pass (kLine) keeps each whole line
  // evict-last in L2 for the value pass, which reads with evict-first
  const uint64_t pol = kLine ? l2_evict_last() : l2_evict_first();
  const bool inter = rs4 == 8;
  auto issue = [&](int t, int slot) {
    const bool v = ok(t);
    const uint4* a = rec + (int64_t)(v ? t : 0) * rs4;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (kLine) cp_async16_128B_pol(ring + (slot * T + tid) * 4 + (u ^ sw), a + u, v, pol);
      else cp_async16_64B(ring + (slot * T + tid) * 4 + (u ^ sw), a + u, v);
    }
    cp_async_commit();
  };
  auto prefetch = [&](int t) {
    if (ok(t)) {
      const uint4* a = rec + (int64_t)t * rs4;
      if (kLine)
        asm volatile("cp.async.bulk.prefetch.L2.global.L2::cache_hint [%0], 128, %1;" ::"l"(a),
                     "l"(pol)
                     : "memory");
      else if (inter)
        asm volatile("cp.async.bulk.prefetch.L2.global.L2::cache_hint [%0], 64, %1;" ::"l"(a),
                     "l"(pol)
                     : "memory");
      else
        asm volatile("cp.async.bulk.prefetch.L2.global [%0], 64;" ::"l"(a) : "memory");
    }
  };
  int i = e0 + tid;
  if (i >= e1) return;
  // q0..q5: the list entries i, i + T, ..., i + 5T
  int q0 = list_at(i), q1 = list_at(i + T), q2 = list_at(i + 2 * T);
  int q3 = list_at(i + 3 * T), q4 = list_at(i + 4 * T), q5 = list_at(i + 5 * T);
  issue(q0, 0);
  float x0 = ok(q0) ? pay(i, q0) : 0.0f;
  issue(q1, 1);
  float x1 = ok(q1) ? pay(i + T, q1) : 0.0f;
  int slot = 0;
  for (; i < e1; i += T) {
    cp_async_wait<1>();               // the slot of entry i has landed
    uint4 w[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) w[u] = ring[(slot * T + tid) * 4 + (u ^ sw)];
    // the slot's words are in registers before the next copy may land in it
    asm volatile("" ::"r"(w[0].x), "r"(w[0].y), "r"(w[0].z), "r"(w[0].w), "r"(w[1].x),
                 "r"(w[1].y), "r"(w[1].z), "r"(w[1].w), "r"(w[2].x), "r"(w[2].y), "r"(w[2].z),
                 "r"(w[2].w), "r"(w[3].x), "r"(w[3].y), "r"(w[3].z), "r"(w[3].w));
    issue(q2, slot);                  // entry i + 2T into the freed slot
    const float x2 = ok(q2) ? pay(i + 2 * T, q2) : 0.0f;
    prefetch(q3);
    if (ok(q0)) f(i, q0, w, x0);
    else record_error(hdr, SDK_ERR_DEVICE_CHECK, tag);
    q0 = q1;
    q1 = q2;
    q2 = q3;
    q3 = q4;
    q4 = q5;
    q5 = list_at(i + 6 * T);
    x0 = x1;
    x1 = x2;
    slot ^= 1;
  }
  cp_async_wait<0>();
}
// for_records without a per-entry value
__device__ __forceinline__ float no_pay(int, int) { return 0.0f; }

// 16 bytes of read-only global memory, not allocated in L1 (the records
// are read once), under the L2 eviction policy pol (createpolicy);
// kLine also asks L2 to fetch the whole 128-byte line.
template <bool kLine>
__device__ __forceinline__ uint4 ld_record16(const uint4* a, uint64_t pol) {
  uint4 v;
  if (kLine)
    asm("ld.global.nc.L1::no_allocate.L2::cache_hint.L2::128B.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
        : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(a), "l"(pol));
  else
    asm("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
        : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(a), "l"(pol));
  return v;
}

// for_records with the records in registers instead of a shared-memory
// ring: each thread holds the records of its next two entries (four
// 16-byte loads each, issued a whole entry ahead of their use) and
// prefetches the records two entries further into L2; no shared-memory
// traffic is spent on moving records.  Same contract as for_records.
// kLine (the key pass over interleaved records): the whole 128-byte line
// is fetched and marked evict-last in L2, so the value record next to the
// key record is still there for the value pass, which reads with
// evict-first (each line is done with after it).
template <bool kLine, class Pay, class F>
__device__ __forceinline__ void for_records_reg(const int32_t* list, int e0, int e1,
                                                const uint4* rec, int rs4, int Nb, WsHeader* hdr,
                                                uint32_t tag, Pay pay, F f) {
  constexpr int T = kAttThreadsReg;
  const int tid = threadIdx.x;
  const uint64_t pol = kLine ? l2_evict_last() : (rs4 == 8 ? l2_evict_first() : 0ull);
  const bool use_pol = kLine || rs4 == 8;
  auto list_at = [&](int i) -> int { return i < e1 ? __ldg(list + i) : -1; };
  auto ok = [&](int t) { return (unsigned)t < (unsigned)Nb; };
  auto load = [&](int t, uint4 (&w)[4]) {
    if (ok(t)) {
      const uint4* a = rec + (int64_t)t * rs4;
      if (use_pol) {
#pragma unroll
        for (int u = 0; u < 4; ++u) w[u] = ld_record16<kLine>(a + u, pol);
      } else {
#pragma unroll
        for (int u = 0; u < 4; ++u)
          asm("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
              : "=r"(w[u].x), "=r"(w[u].y), "=r"(w[u].z), "=r"(w[u].w) : "l"(a + u));
      }
    } else {
#pragma unroll
      for (int u = 0; u < 4; ++u) w[u] = make_uint4(0u, 0u, 0u, 0u);
    }
  };
  auto prefetch = [&](int t) {
    if (ok(t)) {
      const uint4* a = rec + (int64_t)t * rs4;
      if (kLine)
        asm volatile("cp.async.bulk.prefetch.L2.global.L2::cache_hint [%0], 128, %1;" ::"l"(a),
                     "l"(pol)
                     : "memory");
      else
        asm volatile("cp.async.bulk.prefetch.L2.global [%0], 64;" ::"l"(a) : "memory");
    }
  };
  int i = e0 + tid;
  if (i >= e1) return;
  int t0 = list_at(i), t1 = list_at(i + T), t2 = list_at(i + 2 * T), t3 = list_at(i + 3 * T);
  uint4 w0[4], w1[4];
  load(t0, w0);
  float x0 = ok(t0) ? pay(i, t0) : 0.0f;
  load(t1, w1);
  float x1 = ok(t1) ? pay(i + T, t1) : 0.0f;
  prefetch(t2);
  prefetch(t3);
  for (; i < e1; i += 2 * T) {
    if (ok(t0)) f(i, t0, w0, x0);
    else record_error(hdr, SDK_ERR_DEVICE_CHECK, tag);
    t0 = t2;
    load(t0, w0);
    x0 = ok(t0) ? pay(i + 2 * T, t0) : 0.0f;
    t2 = list_at(i + 4 * T);
    prefetch(t2);
    if (i + T >= e1) break;
    if (ok(t1)) f(i + T, t1, w1, x1);
    else record_error(hdr, SDK_ERR_DEVICE_CHECK, tag);
    t1 = t3;
    load(t1, w1);
    x1 = ok(t1) ? pay(i + 3 * T, t1) : 0.0f;
    t3 = list_at(i + 5 * T);
    prefetch(t3);
  }
}

// x = h0 + h1 + h2 in bf16 parts, each the bf16 rounding of what the
// previous parts leave (the remainder is below 2^-24 |x| for normal x)
__device__ __forceinline__ void split3_bf16(float x, uint16_t& h0, uint16_t& h1, uint16_t& h2) {
  const __nv_bfloat16 b0 = __float2bfloat16_rn(x);
  x -= __bfloat162float(b0);
  const __nv_bfloat16 b1 = __float2bfloat16_rn(x);
  x -= __bfloat162float(b1);
  const __nv_bfloat16 b2 = __float2bfloat16_rn(x);
  h0 = __bfloat16_as_ushort(b0);
  h1 = __bfloat16_as_ushort(b1);
  h2 = __bfloat16_as_ushort(b2);
}

// block-wide reduction of one float per thread into s_red[0] (max or sum)
template <bool kMax>
__device__ __forceinline__ float block_reduce(float v, float* s_red) {
  v = kMax ? warp_max(v) : warp_sum(v);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (lane == 0) s_red[warp] = v;
  __syncthreads();
  if (warp == 0) {
    float x = lane < (int)(blockDim.x >> 5) ? s_red[lane] : (kMax ? -INFINITY : 0.0f);
    x = kMax ? warp_max(x) : warp_sum(x);
    if (lane == 0) s_red[32] = x;
  }
  __syncthreads();
  const float r = s_red[32];
  __syncthreads();   // s_red may be reused right away
  return r;
}

// ---- integer softmax (flag SDK_DECODE_INT_SOFTMAX) ------------------------
// Logits of one query head requantised to token-wise INT16 (scale S =
// max |l| / 32767), an integer exponential by I-BERT's second-order
// polynomial exp(p) ~ 0.3585 (p + 1.353)^2 + 0.344 on (-ln 2, 0] with
// exp(x) = 2^-z exp(p), a bit-shift guard that keeps the squares inside
// INT32, an int64 sum and a fixed-point reciprocal (review of "LLM
// Inference in a Flash!", Summary: integer polynomial Softmax on INT16
// requantised inputs with bit-shift overflow guards and fixed-point
// reciprocals; the polynomial is I-BERT's published one).
struct ISoft {
  float S;        // INT16 step of the logits
  int qmax;       // INT16 value of the largest logit
  int sh;         // right shift of q - qmax (overflow guard)
  int q_ln2, q_b, q_c;
};

__device__ __forceinline__ int isoft_q(float l, float S) {
  if (l != l) return -32767;   // NaN: the lowest INT16 value
  const double v = rint((double)l / (double)S);
  return (int)fmin(fmax(v, -32767.0), 32767.0);
}

// constants for logits whose largest magnitude is lmax and largest value lhi
__device__ __forceinline__ ISoft isoft_setup(float lmax, float lhi) {
  ISoft c;
  c.S = lmax > 0.0f ? lmax / 32767.0f : 1.0f;
  c.qmax = isoft_q(lhi, c.S);
  // the smallest shift whose constants keep (p + q_b)^2 + q_c below 2^31
  // (all in fp64; converted to int only once they fit)
  for (c.sh = 0;; ++c.sh) {
    const double sw = ldexp((double)c.S, c.sh);
    const double qb = floor(1.353 / sw);
    const double qc = floor(0.344 / (0.3585 * sw * sw));
    if (qb * qb + qc < 2147483648.0) {
      const double qln2 = floor(0.6931471805599453 / sw);
      c.q_ln2 = qln2 < 1.0 ? 1 : (int)qln2;
      c.q_b = (int)qb;
      c.q_c = (int)qc;
      break;
    }
  }
  return c;
}

// integer exponential of one logit (relative to the largest), < 2^31
__device__ __forceinline__ uint32_t isoft_exp(float l, const ISoft& c) {
  const int x = (isoft_q(l, c.S) - c.qmax) >> c.sh;   // <= 0, arithmetic shift
  const int z = (-x) / c.q_ln2;
  const int pp = x + z * c.q_ln2;
  const long long L = (long long)(pp + c.q_b) * (pp + c.q_b) + c.q_c;
  return z < 31 ? (uint32_t)(L >> z) : 0u;
}

__device__ __forceinline__ unsigned long long block_sum_u64(unsigned long long v,
                                                            unsigned long long* s_red64) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (lane == 0) s_red64[warp] = v;
  __syncthreads();
  if (warp == 0) {
    unsigned long long x = lane < (int)(blockDim.x >> 5) ? s_red64[lane] : 0ull;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    if (lane == 0) s_red64[32] = x;
  }
  __syncthreads();
  const unsigned long long r = s_red64[32];
  __syncthreads();
  return r;
}

template <bool kAll16, bool kCheck, bool kReg>
__global__ void __launch_bounds__(kReg ? kAttThreadsReg : kAttThreads, 1)
    attend_kernel(DecodeParams p, int C) {
  constexpr int kT = kReg ? kAttThreadsReg : kAttThreads;
  pdl_wait();     // nothing global is touched before the previous kernel is done
  pdl_launch();
  extern __shared__ float4 smem4[];
  float* table = reinterpret_cast<float*>(smem4);
  int* siw = reinterpret_cast<int*>(smem4);
  uint4* ring = reinterpret_cast<uint4*>(smem4 + kTable / 4);   // 2 slots x T records
  __shared__ float s_red[33];
  __shared__ float s_val;
  __shared__ float s_val2;
  __shared__ unsigned long long s_red64[33];
  __shared__ unsigned long long s_sum64;
  __shared__ int s_float;
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  const int n = p.n, tid = threadIdx.x;
  const int r = blockIdx.x / C;
  const int rank = (int)cluster.block_rank();
  const int b = r / p.Hq, h = r % p.Hq, kvh = h / p.g;
  sdk_select_state* st = p.st + r;
  // context-sharded stages take the head's local selected count from the
  // state (the rest of the selection is on the other ranks)
  const int Nb = p.lens[b];
  const int k = p.att_mode ? (int)min(__ldcg(&st->n_sel), (uint32_t)Nb) : p.kcnt[b];
  const int Dr = p.att_mode ? k : p.dcnt[b];
  const int s0 = (int)((int64_t)k * rank / C), s1 = (int)((int64_t)k * (rank + 1) / C);
  const int c0 = k + (int)((int64_t)(Dr - k) * rank / C);
  const int c1 = k + (int)((int64_t)(Dr - k) * (rank + 1) / C);
  const int64_t head = (int64_t)b * p.Hkv + kvh;
  const uint4* krec = reinterpret_cast<const uint4*>(p.k_full + head * p.cap * p.rs);
  const uint4* vrec = reinterpret_cast<const uint4*>(p.v_full + head * p.cap * p.rs);
  const int rs4 = p.rs / 4;
  const int32_t* list = p.list + (int64_t)r * p.L;
  float* ss = p.sel_score + (int64_t)r * p.L;
  // the records of list entries [a0, a1): in registers (kReg) or through
  // the shared-memory ring
  auto recs = [&](auto line, int a0, int a1, const uint4* rc, uint32_t tag, auto pay, auto f) {
    constexpr bool kL = decltype(line)::value;
    if constexpr (kReg) for_records_reg<kL>(list, a0, a1, rc, rs4, Nb, p.hdr, tag, pay, f);
    else for_records<kL>(list, a0, a1, rc, rs4, Nb, p.hdr, tag, ring, pay, f);
  };
  const uint32_t* keys = p.keys + (int64_t)r * p.L;
  const float scale = p.scale;
  const int khigh = p.khigh;
  uint32_t maxidx = 0u;

  float m = -INFINITY;
  const bool isoft = p.isoft != 0;
  ISoft ic;
  unsigned long long recip = 0ull, etot = 0ull;
  float ztot = 0.0f;
  if (p.att_mode == 2) {
    // context-sharded, second half: the softmax statistics of every rank
    // (mz [world][R][2]: the rank's largest logit and its sum of
    // exp(s - that) for this head) give this head's m and z
    const float* mz = reinterpret_cast<const float*>(p.shard_in);
    for (int w = 0; w < p.world; ++w) m = fmaxf(m, __ldcg(mz + ((int64_t)w * p.R + r) * 2));
    for (int w = 0; w < p.world; ++w) {
      const float mw = __ldcg(mz + ((int64_t)w * p.R + r) * 2);
      const float zw = __ldcg(mz + ((int64_t)w * p.R + r) * 2 + 1);
      if (mw > -INFINITY && zw > 0.0f) ztot += zw * expf(mw - m);
    }
    if (tid == 0) s_float = 0;
    cluster.sync();
  } else {
  // ---- phase 1: stage QD[r], rescore the own selected entries
  stage_table(table, p.qd + (int64_t)r * n, n);
  __syncthreads();
  float smax = -INFINITY, zrun = 0.0f;     // online softmax of this thread
  float smin = INFINITY;                   // for the integer softmax's scale
  auto key_pass = [&](auto line, auto f) { recs(line, s0, s1, krec, 0x30000000u | r, no_pay, f); };
  auto rescore = 
              [&](int i, int t, const uint4 (&w)[4], float) {
                float s = 0.0f;
#pragma unroll
                for (int u = 0; u < 16; ++u) {
                  if (!kAll16 && u >= khigh) break;
                  const uint32_t wd = (u & 3) == 0 ? w[u >> 2].x : (u & 3) == 1 ? w[u >> 2].y
                                    : (u & 3) == 2 ? w[u >> 2].z : w[u >> 2].w;
                  const uint32_t idx = word_idx(wd);
                  if (kCheck) maxidx = max(maxidx, idx);
                  s = fmaf(word_coef(wd), table[idx], s);
                }
                s *= scale;
                ss[i] = s;
                smin = fminf(smin, s);
                if (s > smax) {
                  zrun = zrun * expf(smax - s) + 1.0f;
                  smax = s;
                } else {
                  zrun += expf(s - smax);
                }
              };
  if (p.rs == 2 * kAtoms) key_pass(std::true_type{}, rescore);
  else key_pass(std::false_type{}, rescore);
  m = block_reduce<true>(smax, s_red);
  if (tid == 0) s_val = m;
  cluster.sync();
  m = -INFINITY;
  for (int cc = 0; cc < C; ++cc) m = fmaxf(m, *cluster.map_shared_rank(&s_val, cc));
  if (rank == 0 && tid == 0 && m > -INFINITY) st->max_score = score_key(m);
  if (p.full && st->n_comp > 0u) m = fmaxf(m, scale * key_score(st->max_comp));

  if (!isoft) {
    // z: the own selected entries (rescaled to m) and complement entries
    float z = smax > -INFINITY ? zrun * expf(smax - m) : 0.0f;
#pragma unroll 4
    for (int i = c0 + tid; i < c1; i += kT) {
      const int t = list[i];
      if ((unsigned)t < (unsigned)Nb) z += expf(scale * key_score(keys[t]) - m);
    }
    z = block_reduce<false>(z, s_red);
    cluster.sync();   // every CTA has read s_val of phase 1
    if (tid == 0) {
      s_val = z;
      s_float = 0;
    }
    cluster.sync();
    for (int cc = 0; cc < C; ++cc) ztot += *cluster.map_shared_rank(&s_val, cc);
  } else {
    // the smallest logit of the domain (own selected and complement
    // entries), then the INT16 scale, the integer exponentials and their sum
#pragma unroll 4
    for (int i = c0 + tid; i < c1; i += kT) {
      const int t = list[i];
      if ((unsigned)t < (unsigned)Nb) smin = fminf(smin, scale * key_score(keys[t]));
    }
    const float mn = -block_reduce<true>(-smin, s_red);
    cluster.sync();   // every CTA has read s_val of phase 1
    if (tid == 0) s_val2 = mn;
    cluster.sync();
    float lo = INFINITY;
    for (int cc = 0; cc < C; ++cc) lo = fminf(lo, *cluster.map_shared_rank(&s_val2, cc));
    const float hi_abs = m > -INFINITY ? fabsf(m) : 0.0f;
    const float lo_abs = lo < INFINITY ? fabsf(lo) : 0.0f;
    ic = isoft_setup(fmaxf(hi_abs, lo_abs), m > -INFINITY ? m : 0.0f);
    unsigned long long e = 0ull;
    for (int i = s0 + tid; i < s1; i += kT) e += isoft_exp(ss[i], ic);
#pragma unroll 4
    for (int i = c0 + tid; i < c1; i += kT) {
      const int t = list[i];
      if ((unsigned)t < (unsigned)Nb) e += isoft_exp(scale * key_score(keys[t]), ic);
    }
    e = block_sum_u64(e, s_red64);
    if (tid == 0) {
      s_sum64 = e;
      s_float = 0;
    }
    cluster.sync();
    for (int cc = 0; cc < C; ++cc) etot += *cluster.map_shared_rank(&s_sum64, cc);
    recip = etot > 0ull ? (1ull << 61) / etot : 0ull;
    ztot = (float)etot;
  }
  if (p.att_mode == 1) {
    // context-sharded, first half: this rank's statistics of the head go to
    // mz [R][2] (gathered over the ranks); the cluster's shared memory stays
    // until every CTA has read it
    if (kCheck && maxidx >= (uint32_t)n) record_error(p.hdr, SDK_ERR_DEVICE_CHECK, maxidx);
    if (rank == 0 && tid == 0) {
      float* mz = reinterpret_cast<float*>(p.hist2) + p.R + 2 * r;
      mz[0] = m;
      mz[1] = ztot;
    }
    cluster.sync();
    return;
  }
  }   // phase 1
  const float invz = 1.0f / ztot;

  // ---- phase 2: scatter p c^V into the weight tile
  auto phase2 = [&](auto fl) {
    constexpr bool kFloat = decltype(fl)::value;
    {
      uint4* t4 = reinterpret_cast<uint4*>(smem4);
      for (int i = tid; i < kTable / 4; i += kT) t4[i] = make_uint4(0u, 0u, 0u, 0u);
    }
    __syncthreads();
    // fixed point: p already carries the 2^20 scale
    const float pscale = kFloat ? invz : invz * kFixScale;
    float absum = 0.0f;
    // integer softmax: P in Q30 from the integer exponential and the
    // fixed-point reciprocal, then the tile's scale (2^20 or 1)
    const float qscale = kFloat ? 9.313225746154785e-10f : 9.765625e-4f;   // 2^-30, 2^-10
    auto scatter = [&](float lg, const uint4 (&w)[4]) {
      const float pt =
          isoft ? (float)(((unsigned long long)isoft_exp(lg, ic) * recip) >> 31) * qscale
                : expf(lg - m) * pscale;
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const uint32_t wd = (u & 3) == 0 ? w[u >> 2].x : (u & 3) == 1 ? w[u >> 2].y
                          : (u & 3) == 2 ? w[u >> 2].z : w[u >> 2].w;
        const uint32_t idx = word_idx(wd);
        if (kCheck) maxidx = max(maxidx, idx);
        const float v = pt * word_coef(wd);
        if constexpr (kFloat) {
          atomicAdd(&table[idx], v);
        } else {
          absum += fabsf(v);
          atomicAdd(&siw[idx], __float2int_rn(v));
        }
      }
    };
    // the logits load with the records: the rescored ones, and with the
    // flag the complement's scale * s_lo
    recs(std::false_type{}, s0, s1, vrec, 0x31000000u | r,
                [&](int i, int) { return ss[i]; },
                [&](int, int, const uint4 (&w)[4], float lg) { scatter(lg, w); });
    if (p.full)
      recs(std::false_type{}, c0, c1, vrec, 0x32000000u | r,
                  [&](int, int t) { return scale * key_score(keys[t]); },
                  [&](int, int, const uint4 (&w)[4], float lg) { scatter(lg, w); });
    // int32 range guard (also catches NaN): sum |p c| * 2^20 < 2^30
    if (!kFloat && !(absum < 1073741824.0f)) s_float = 1;
    __syncthreads();
  };
  phase2(std::false_type{});
  if (s_float) phase2(std::true_type{});
  if (kCheck && maxidx >= (uint32_t)n) record_error(p.hdr, SDK_ERR_DEVICE_CHECK, maxidx);

  // ---- phase 3: sum the cluster's tiles over this CTA's slice of atoms,
  // in groups of 4 atoms; a group's loads from all C tiles are in flight
  // before any is summed
  cluster.sync();
  const int ng = (n + 3) >> 2;
  const int g0 = (int)((int64_t)ng * rank / C), g1 = (int)((int64_t)ng * (rank + 1) / C);
  // w as three bf16 parts (the operand layout of the tensor-core w D_V)
  const int64_t plane = (int64_t)p.R * n;
  uint16_t* gw = p.w + (int64_t)r * n;
  const int4* tiles[8];
  bool isf[8];
#pragma unroll
  for (int cc = 0; cc < 8; ++cc) {
    if (cc < C) {
      tiles[cc] = reinterpret_cast<const int4*>(cluster.map_shared_rank(siw, cc));
      isf[cc] = *cluster.map_shared_rank(&s_float, cc) != 0;
    }
  }
  for (int g = g0 + tid; g < g1; g += kT) {
    int4 v[8];
#pragma unroll
    for (int cc = 0; cc < 8; ++cc)
      if (cc < C) v[cc] = tiles[cc][g];
    float sum[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int cc = 0; cc < 8; ++cc) {
      if (cc >= C) break;
      const int vv[4] = {v[cc].x, v[cc].y, v[cc].z, v[cc].w};
#pragma unroll
      for (int u = 0; u < 4; ++u) sum[u] += isf[cc] ? __int_as_float(vv[u]) : (float)vv[u] * kFixInv;
    }
    uint16_t parts[3][4];
#pragma unroll
    for (int u = 0; u < 4; ++u) split3_bf16(sum[u], parts[0][u], parts[1][u], parts[2][u]);
    if (4 * g + 3 < n && (n & 3) == 0) {
#pragma unroll
      for (int s3 = 0; s3 < 3; ++s3)
        *reinterpret_cast<uint2*>(gw + s3 * plane + 4 * g) =
            make_uint2(parts[s3][0] | ((uint32_t)parts[s3][1] << 16),
                       parts[s3][2] | ((uint32_t)parts[s3][3] << 16));
    } else {
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (4 * g + u < n)
#pragma unroll
          for (int s3 = 0; s3 < 3; ++s3) gw[s3 * plane + 4 * g + u] = parts[s3][u];
    }
  }
  if (rank == 0 && tid == 0) {
    st->z = ztot;
    if (isoft) {
      st->isoft_sum[0] = (uint32_t)etot;
      st->isoft_sum[1] = (uint32_t)(etot >> 32);
      st->isoft_shift = (uint32_t)ic.sh;
    }
  }
  cluster.sync();
}

// --------------------------------------------------------------- out_kernel
// out[r][c] += sum_a w[r][a] D_V[a][c] over kGvTiles consecutive atom tiles
// of kGvAtoms atoms and RB row blocks of 32 rows.  All value tiles of the
// CTA are requested at once with cp.async (bf16 [atom][D], natural layout:
// the column loads below are contiguous); each tile's weights are staged
// fp32 [a][32] (4-row groups XOR-swizzled by a).  Lane (tc, tr) of warp w
// of a row block owns columns 32w + 4tc .. +3 and rows 8tr .. 8tr+7 (32
// accumulators over the CTA's atoms): per atom one 8-byte value load and two
// broadcast weight loads feed 32 FMAs.  The partial sums are added into
// `out` (zeroed by qd_kernel) with one vector reduction per row.
// w[r][a] from its three bf16 parts
__device__ __forceinline__ float w_at(const DecodeParams& p, int r, int a) {
  const int64_t plane = (int64_t)p.R * p.n, o = (int64_t)r * p.n + a;
  const float w0 = __uint_as_float((uint32_t)__ldg(p.w + o) << 16);
  const float w1 = __uint_as_float((uint32_t)__ldg(p.w + plane + o) << 16);
  const float w2 = __uint_as_float((uint32_t)__ldg(p.w + 2 * plane + o) << 16);
  return w0 + (w1 + w2);
}
constexpr int out_smem_bytes(int d, int rb, int tiles) {
  return tiles * kGvAtoms * d * 2 + rb * kGvAtoms * 32 * 4;
}

template <int D, int RB, int kGvTiles>
__global__ void __launch_bounds__(D * RB) out_kernel(DecodeParams p) {
  pdl_wait();     // nothing global is touched before the previous kernel is done
  pdl_launch();
  constexpr int kThreads = D * RB;                // D/32 warps per row block
  constexpr int kChunks = D / 8;
  extern __shared__ uint4 out_smem[];
  uint4* Vt = out_smem;                           // [atom][chunk], kGvTiles tiles
  float* Ws = reinterpret_cast<float*>(out_smem + kGvTiles * kGvAtoms * kChunks);  // [rb][a][32]
  const int n = p.n, R = p.R, tid = threadIdx.x;
  const int a0 = blockIdx.x * (kGvTiles * kGvAtoms);
  const int r0 = blockIdx.y * (32 * RB);
  for (int e = tid; e < kGvTiles * kGvAtoms * kChunks; e += kThreads) {
    const int a = e / kChunks, c = e % kChunks;
    const bool v = a0 + a < n;
    const uint4* src = reinterpret_cast<const uint4*>(p.dv + (int64_t)(v ? a0 + a : 0) * D) + c;
    cp_async16(Vt + a * kChunks + c, src, v);
  }
  cp_async_commit();
  const int lane = tid & 31, warp = tid >> 5;
  const int rb = warp / (D / 32), wc = warp % (D / 32);
  const int tc = lane & 7, tr = lane >> 3;
  const int cc = 32 * wc + 4 * tc;
  float acc[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int u = 0; u < 4; ++u) acc[i][u] = 0.0f;
  for (int tile = 0; tile < kGvTiles; ++tile) {
    const int ta0 = a0 + tile * kGvAtoms;
    if (ta0 >= n) break;
    if (tile) __syncthreads();                    // previous weights consumed
    // weights of this tile: lanes along atoms (coalesced), all of a
    // thread's loads in flight before its first store
    constexpr int kW = RB * kGvAtoms * 32;
    constexpr int kWPer = (kW + kThreads - 1) / kThreads;
    for (int e0 = tid; e0 < kW; e0 += kWPer * kThreads) {
      float v[kWPer];
#pragma unroll
      for (int u = 0; u < kWPer; ++u) {
        const int e = e0 + u * kThreads;
        const int a = e % kGvAtoms, rr = e / kGvAtoms;
        v[u] = (e < kW && r0 + rr < R && ta0 + a < n) ? w_at(p, r0 + rr, ta0 + a) : 0.0f;
      }
#pragma unroll
      for (int u = 0; u < kWPer; ++u) {
        const int e = e0 + u * kThreads;
        if (e >= kW) break;
        const int a = e % kGvAtoms, rr = e / kGvAtoms;
        Ws[((rr >> 5) * kGvAtoms + a) * 32 + qswz(a, rr & 31)] = v[u];
      }
    }
    if (tile == 0) cp_async_wait<0>();
    __syncthreads();
    const uint4* Vtile = Vt + tile * kGvAtoms * kChunks;
    const float* Wb = Ws + rb * kGvAtoms * 32;
#pragma unroll 4
    for (int a = 0; a < kGvAtoms; ++a) {
      const uint2 vv = reinterpret_cast<const uint2*>(Vtile + a * kChunks)[cc >> 2];
      const float4 wa = *reinterpret_cast<const float4*>(Wb + a * 32 + (((2 * tr) ^ (a & 7)) << 2));
      const float4 wb = *reinterpret_cast<const float4*>(Wb + a * 32 + (((2 * tr + 1) ^ (a & 7)) << 2));
      const float dv[4] = {bf16_lo(vv.x), bf16_hi(vv.x), bf16_lo(vv.y), bf16_hi(vv.y)};
      const float wr[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int u = 0; u < 4; ++u) acc[i][u] = fmaf(wr[i], dv[u], acc[i][u]);
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int r = r0 + rb * 32 + 8 * tr + i;
    if (r >= R) continue;
    float* dst = p.out + (int64_t)r * D + cc;
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(dst), "f"(acc[i][0]),
                 "f"(acc[i][1]), "f"(acc[i][2]), "f"(acc[i][3])
                 : "memory");
  }
}

// --------------------------------------------------------------- launcher
static size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

sdk_decode_layout decode_layout(int B, int Hq, int d, int n, int64_t L) {
  sdk_decode_layout l;
  const size_t R = (size_t)B * Hq;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = align_up(off + bytes, 256);
    return o;
  };
  (void)d;
  L = (L + 3) & ~(int64_t)3;   // 16-byte aligned rows
  l.row = (size_t)L;
  l.header = take(sizeof(WsHeader));
  l.qd = take(R * n * 4);
  l.keys = take(R * L * 4);
  l.hist1 = take(R * 4096 * 4);
  l.hist2 = take(R * 4096 * 4);
  l.state = take(R * sizeof(sdk_select_state));
  l.list = take(R * L * 4);
  l.cand_t = take(R * L * 4);
  l.cand_key = take(R * L * 4);
  l.sel_score = take(R * L * 4);
  l.w = take(3 * R * n * 2);
  l.part = take(0);
  l.total = off;
  return l;
}

static int grid_for(int64_t work, int64_t per_cta, int cap_ctas) {
  int64_t g = (work + per_cta - 1) / per_cta;
  if (g < 1) g = 1;
  if (g > cap_ctas) g = cap_ctas;
  return (int)g;
}

// CTAs for a segment scan (klow, pass 2) over `total` tokens of R heads with
// a start-up cost of `a` tokens per head touched: up to g CTAs splitting the
// virtual space, or the largest multiple of R below g, whose boundaries fall
// on head starts when the heads are equally long (no CTA pays a second
// start-up), whichever gives the smaller cost per CTA.
static int scan_grid(int64_t total, int64_t R, int64_t a, int64_t per_cta, int sms) {
  const int g = grid_for(total, per_cta, sms);
  if (R > g) return g;
  const int64_t ga = R * (g / R);
  const double c_split = (double)(total + a * (g + R)) / g;
  const double c_aligned = (double)total / ga + (double)a;
  return c_aligned <= c_split ? (int)ga : g;
}

// Optional launch with programmatic stream serialization (the kernel may
// start while the previous one drains; every decode kernel waits for it
// before touching memory).  Off by default: measured on B200 it made the
// 32-layer 256K-token step slower (early-resident CTAs of the next kernel
// hold SM resources); SDK_DECODE_PDL=1 in the environment turns it on.
static bool pdl_enabled() {
  static int on = -1;
  if (on < 0) {
    const char* v = getenv("SDK_DECODE_PDL");
    on = (v != nullptr && v[0] == '1') ? 1 : 0;
  }
  return on == 1;
}

// The attention kernel streams records through a shared-memory ring unless
// SDK_ATTEND_RING=0 (then through registers; measured slower at 256K: 67.8
// against 62.5 us per launch).
static bool attend_ring() {
  static int on = -1;
  if (on < 0) {
    const char* v = getenv("SDK_ATTEND_RING");
    on = (v != nullptr && v[0] == '0') ? 0 : 1;
  }
  return on == 1;
}

// Entries of the Klow scan's per-segment buffer of selected tokens in the
// bracket path (candidates: half as many); SDK_KLOW_BUF overrides.
static int klow_above_buf() {
  static int v = -1;
  if (v < 0) {
    const char* e = getenv("SDK_KLOW_BUF");
    int x = e != nullptr ? atoi(e) : 0;
    v = (x >= 256 && x <= kKlowAboveBuf) ? (x & ~255) : kKlowAboveBuf;
  }
  return v;
}

// QD on the tensor cores (three bf16 parts of q) unless SDK_DECODE_QD_TC=0.
static bool qd_tensor_cores() {
  static int on = -1;
  if (on < 0) {
    const char* v = getenv("SDK_DECODE_QD_TC");
    on = (v != nullptr && v[0] == '0') ? 0 : 1;
  }
  return on == 1;
}

// w D_V on the tensor cores (three bf16 parts of w) unless SDK_DECODE_OUT_TC=0.
static bool out_tensor_cores() {
  static int on = -1;
  if (on < 0) {
    const char* v = getenv("SDK_DECODE_OUT_TC");
    on = (v != nullptr && v[0] == '0') ? 0 : 1;
  }
  return on == 1;
}

// With SDK_DEBUG=1 in the environment a failed launch is reported on
// stderr with the CUDA error (the call still returns SDK_ERR_CUDA).
static bool debug_launches() {
  static int on = -1;
  if (on < 0) {
    const char* v = getenv("SDK_DEBUG");
    on = (v != nullptr && v[0] == '1') ? 1 : 0;
  }
  return on == 1;
}

template <class... KArgs, class... Args>
static cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t stream, unsigned cluster, Args... args);

template <class... KArgs, class... Args>
static cudaError_t launch_checked(const char* name, void (*kern)(KArgs...), dim3 grid, dim3 block,
                                  size_t smem, cudaStream_t stream, unsigned cluster,
                                  Args... args) {
  const cudaError_t e = launch_pdl(kern, grid, block, smem, stream, cluster, args...);
  if (debug_launches()) {
    const cudaError_t e2 = e != cudaSuccess ? e : cudaPeekAtLastError();
    if (e2 != cudaSuccess)
      fprintf(stderr, "sdk: launch of %s (grid %u, block %u, smem %zu, cluster %u): %s\n", name,
              grid.x, block.x, smem, cluster, cudaGetErrorString(e2));
  }
  return e;
}

template <class... KArgs, class... Args>
static cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t stream, unsigned cluster, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute at[2];
  int na = 0;
  if (pdl_enabled()) {
    at[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  if (cluster > 1) {
    at[na].id = cudaLaunchAttributeClusterDimension;
    at[na].val.clusterDim.x = cluster;
    at[na].val.clusterDim.y = 1;
    at[na].val.clusterDim.z = 1;
    ++na;
  }
  cfg.attrs = at;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

// ---- attention-kernel timing (sdk_timing_enable / sdk_timing_read) -------
namespace {
constexpr int kTimingDevices = 64;
std::atomic<bool> g_timing_on{false};
std::mutex g_timing_mu;
struct TimingPool {
  cudaEvent_t ev[SDK_TIMING_SLOTS][2];
  bool made = false;
  int used = 0;
};
TimingPool g_timing[kTimingDevices];

}  // namespace

// The event pair of the next slot of the current device (nulls when timing
// is off, or was not turned on for this device).
void timing_slot(cudaEvent_t* e0, cudaEvent_t* e1) {
  *e0 = *e1 = nullptr;
  if (!g_timing_on.load(std::memory_order_acquire)) return;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kTimingDevices) return;
  std::lock_guard<std::mutex> lock(g_timing_mu);
  TimingPool& tp = g_timing[dev];
  if (!tp.made) return;   // enabled on another device
  const int i = tp.used % SDK_TIMING_SLOTS;
  ++tp.used;
  *e0 = tp.ev[i][0];
  *e1 = tp.ev[i][1];
}
// Records e on stream; inside a stream capture as an external record (an
// event-record node of the graph, executed by every replay), which a plain
// record there is not.
cudaError_t timing_record(cudaEvent_t e, cudaStream_t stream) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(stream, &cs) != cudaSuccess) return cudaErrorUnknown;
  return cs == cudaStreamCaptureStatusActive
             ? cudaEventRecordWithFlags(e, stream, cudaEventRecordExternal)
             : cudaEventRecord(e, stream);
}


// The current device's events are made here, outside any stream capture.
sdk_status timing_enable(bool on) {
  std::lock_guard<std::mutex> lock(g_timing_mu);
  if (on) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kTimingDevices)
      return SDK_ERR_CUDA;
    TimingPool& tp = g_timing[dev];
    if (!tp.made) {
      for (int i = 0; i < SDK_TIMING_SLOTS; ++i)
        for (int j = 0; j < 2; ++j)
          if (cudaEventCreate(&tp.ev[i][j]) != cudaSuccess) return SDK_ERR_CUDA;
      tp.made = true;
    }
    tp.used = 0;
  }
  g_timing_on.store(on, std::memory_order_release);
  return SDK_OK;
}

int timing_read(float* ms_out, int max_n) {
  if (ms_out == nullptr || max_n < 0) return -1;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kTimingDevices) return -1;
  std::lock_guard<std::mutex> lock(g_timing_mu);
  TimingPool& tp = g_timing[dev];
  if (!tp.made) return 0;
  int n = tp.used < SDK_TIMING_SLOTS ? tp.used : SDK_TIMING_SLOTS;
  if (n > max_n) n = max_n;
  for (int i = 0; i < n; ++i) {
    if (cudaEventSynchronize(tp.ev[i][1]) != cudaSuccess ||
        cudaEventElapsedTime(&ms_out[i], tp.ev[i][0], tp.ev[i][1]) != cudaSuccess) {
      cudaGetLastError();   // not sticky: leave no error for the next call
      return -1;
    }
  }
  return n;
}

sdk_status launch_decode(DecodeParams p, cudaStream_t stream, int shard_stage, int rank_id) {
  const int sms = num_sms();
  static unsigned long long attr_set = 0ull;
  if (device_needs_setup(&attr_set)) {
    cudaFuncSetAttribute(klow_kernel<false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         kKlowSmemHist);
    cudaFuncSetAttribute(klow_kernel<false, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         kKlowSmemHist);
    cudaFuncSetAttribute(klow_kernel<true, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         kKlowSmemBracket);
    cudaFuncSetAttribute(klow_kernel<true, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         kKlowSmemBracket);
    cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSelSmem);
    cudaFuncSetAttribute(sample_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSampleSmem);
    cudaFuncSetAttribute(pass2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kPass2Smem);
    cudaFuncSetAttribute(final_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         2 * kFinalStage * 4);
    cudaFuncSetAttribute(qd_kernel<128, 2, 4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         qd_smem_bytes(128, 2, 4));
    cudaFuncSetAttribute(qd_kernel<64, 2, 4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         qd_smem_bytes(64, 2, 4));
    cudaFuncSetAttribute(out_kernel<128, 2, 4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         out_smem_bytes(128, 2, 4));
    cudaFuncSetAttribute(out_kernel<64, 2, 4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         out_smem_bytes(64, 2, 4));

    cudaFuncSetAttribute(attend_kernel<true, true, false>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, kAttSmem);
    cudaFuncSetAttribute(attend_kernel<true, false, false>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, kAttSmem);
    cudaFuncSetAttribute(attend_kernel<false, true, false>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, kAttSmem);
    cudaFuncSetAttribute(attend_kernel<false, false, false>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, kAttSmem);
    cudaFuncSetAttribute(attend_kernel<true, true, true>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, kAttSmemReg);
    cudaFuncSetAttribute(attend_kernel<true, false, true>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, kAttSmemReg);
    cudaFuncSetAttribute(attend_kernel<false, true, true>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, kAttSmemReg);
    cudaFuncSetAttribute(attend_kernel<false, false, true>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, kAttSmemReg);
    device_setup_done(&attr_set);
  }
  cudaError_t e = cudaSuccess;
  // GEMV shapes: up to 32 query rows one tile x one row block per CTA,
  // above that four tiles x two row blocks (the staged rows are reused)
  const bool wide = p.R > 32;
  const int gv_tiles = wide ? 4 : 1, gv_rb = wide ? 2 : 1;
  const dim3 gv_grid((p.n + gv_tiles * kGvAtoms - 1) / (gv_tiles * kGvAtoms),
                     (p.R + 32 * gv_rb - 1) / (32 * gv_rb));
  auto run = [&](int part) -> sdk_status {
  switch (part) {
  case 0: {   // QD and the Klow scan
  bool qd_tc = false;
  if (qd_tensor_cores()) {
    const sdk_status st = launch_qd_tc(p, stream, &qd_tc);
    if (st != SDK_OK) return st;
  }
  if (!qd_tc) {
    const size_t sm = qd_smem_bytes(p.d, gv_rb, gv_tiles);
    const unsigned th = 64 * gv_tiles * gv_rb;
    if (p.d == 128) {
      e = wide ? launch_checked("qd_kernel", qd_kernel<128, 2, 4>, gv_grid, dim3(th), sm, stream, 1, p)
               : launch_checked("qd_kernel", qd_kernel<128, 1, 1>, gv_grid, dim3(th), sm, stream, 1, p);
    } else {
      e = wide ? launch_checked("qd_kernel", qd_kernel<64, 2, 4>, gv_grid, dim3(th), sm, stream, 1, p)
               : launch_checked("qd_kernel", qd_kernel<64, 1, 1>, gv_grid, dim3(th), sm, stream, 1, p);
    }
    if (e != cudaSuccess) return SDK_ERR_CUDA;
  }
  {
    const int g = scan_grid(p.tok_off[p.B], p.R, kKlowSegCost, 2048, sms);
    const int vec = (p.cap % 4 == 0) && ((reinterpret_cast<uintptr_t>(p.k_lo) & 15u) == 0u);
    if (p.bracket) {
      e = launch_checked("sample_kernel", sample_kernel, dim3(p.R), dim3(kSampleThreads), (size_t)kSampleSmem, stream,
                     1, p);
      if (e != cudaSuccess) return SDK_ERR_CUDA;
      p.klow_buf = klow_above_buf();
      e = launch_checked("klow_kernel", p.n < kTable ? klow_kernel<true, true> : klow_kernel<true, false>,
                         dim3(g), dim3(kKlowThreads),
                         (size_t)kTable * 4 + (size_t)p.klow_buf * 8,
                     stream, 1, p, vec);
    } else {
      e = launch_checked("klow_kernel", p.n < kTable ? klow_kernel<false, true> : klow_kernel<false, false>,
                         dim3(g), dim3(kKlowThreads), (size_t)kKlowSmemHist,
                     stream, 1, p, vec);
    }
    if (e != cudaSuccess) return SDK_ERR_CUDA;
  }
  return SDK_OK;
  }
  case 1: {   // pass 2 of the selection (radix path only)
    if (p.bracket) return SDK_OK;
    const int g = scan_grid(p.tok_off[p.B], p.R, kPass2SegCost, 8192, sms);
    e = launch_checked("pass2_kernel", pass2_kernel, dim3(g), dim3(kP2Threads), (size_t)kPass2Smem, stream, 1, p);
    return e == cudaSuccess ? SDK_OK : SDK_ERR_CUDA;
  }
  case 2:     // the final selection (whole context)
    if (p.bracket)
      e = launch_checked("select_kernel", select_kernel, dim3(p.R), dim3(kSelThreads), (size_t)kSelSmem, stream, 1, p);
    else
      e = launch_checked("final_kernel", final_kernel, dim3(p.R), dim3(kScanThreads), (size_t)2 * kFinalStage * 4,
                     stream, 1, p);
    return e == cudaSuccess ? SDK_OK : SDK_ERR_CUDA;
  case 3: {   // attend
  {
    cudaEvent_t t0 = nullptr, t1 = nullptr;
    timing_slot(&t0, &t1);
    if (t0 != nullptr && timing_record(t0, stream) != cudaSuccess) return SDK_ERR_CUDA;
    // one cluster of C CTAs per query head, C a power of two <= 8 while the
    // clusters fit the SMs and every CTA keeps >= 1024 entries
    int64_t dmax = 0;
    for (int b = 0; b < p.B; ++b) dmax = p.dcnt[b] > dmax ? p.dcnt[b] : dmax;
    int C = 1;
    while (C < 8 && (int64_t)p.R * C * 2 <= sms && dmax / (2 * C) >= 1024) C *= 2;
    const bool all16 = p.khigh == kAtoms, check = p.n < kTable;
    const bool reg = !attend_ring();
    auto kern = reg ? (all16 ? (check ? attend_kernel<true, true, true> : attend_kernel<true, false, true>)
                             : (check ? attend_kernel<false, true, true> : attend_kernel<false, false, true>))
                    : (all16 ? (check ? attend_kernel<true, true, false> : attend_kernel<true, false, false>)
                             : (check ? attend_kernel<false, true, false> : attend_kernel<false, false, false>));
    e = launch_checked("attend_kernel", kern, dim3((unsigned)(p.R * C)), dim3(reg ? kAttThreadsReg : kAttThreads),
                   (size_t)(reg ? kAttSmemReg : kAttSmem), stream, (unsigned)C, p, C);
    if (e != cudaSuccess) return SDK_ERR_CUDA;
    if (t1 != nullptr && timing_record(t1, stream) != cudaSuccess) return SDK_ERR_CUDA;
  }
  return SDK_OK;
  }
  default: {  // w D_V
  // w D_V on the tensor cores (the CUDA-core kernel where they are off or
  // the shapes do not allow tensor maps)
  bool out_tc = false;
  if (out_tensor_cores()) {
    const sdk_status st = launch_out_tc(p, stream, &out_tc);
    if (st != SDK_OK) return st;
  }
  if (!out_tc) {
    if (wide) {
      const size_t sm = out_smem_bytes(p.d, gv_rb, gv_tiles);
      e = p.d == 128 ? launch_checked("out_kernel", out_kernel<128, 2, 4>, gv_grid, dim3(256), sm, stream, 1, p)
                     : launch_checked("out_kernel", out_kernel<64, 2, 4>, gv_grid, dim3(128), sm, stream, 1, p);
    } else {
      // up to 32 rows: 64 atoms per CTA (measured faster than 128 or 256)
      const size_t sm = out_smem_bytes(p.d, 1, 1);
      e = p.d == 128 ? launch_checked("out_kernel", out_kernel<128, 1, 1>, gv_grid, dim3(128), sm, stream, 1, p)
                     : launch_checked("out_kernel", out_kernel<64, 1, 1>, gv_grid, dim3(64), sm, stream, 1, p);
    }
    if (e != cudaSuccess) return SDK_ERR_CUDA;
  }
  return SDK_OK;
  }
  }
  };
  if (shard_stage == 0) {
    for (int part = 0; part < 5; ++part) {
      const sdk_status st = run(part);
      if (st != SDK_OK) return st;
    }
  } else {
    // context-sharded stages (sdk_decode_attn_shard): 1 QD + Klow scan;
    // 2 pass 2; 3 third digit; 4 key and ties; 5 local selection and
    // attend's first half; 6 attend's second half and w D_V
    sdk_status st = SDK_OK;
    switch (shard_stage) {
      case 1: st = run(0); break;
      case 2: st = run(1); break;
      case 3:
        e = launch_checked("shard_digit3_kernel", shard_digit3_kernel, dim3(p.R), dim3(kScanThreads), 0, stream, 1, p);
        st = e == cudaSuccess ? SDK_OK : SDK_ERR_CUDA;
        break;
      case 4:
        e = launch_checked("shard_ties_kernel", shard_ties_kernel, dim3(p.R), dim3(kScanThreads), 0, stream, 1, p);
        st = e == cudaSuccess ? SDK_OK : SDK_ERR_CUDA;
        break;
      case 5:
        e = launch_checked("shard_select_kernel", shard_select_kernel, dim3(p.R), dim3(kScanThreads), 0, stream, 1, p,
                       reinterpret_cast<const uint32_t*>(p.shard_in), rank_id);
        if (e != cudaSuccess) return SDK_ERR_CUDA;
        p.att_mode = 1;
        st = run(3);
        p.att_mode = 0;
        break;
      case 6:
        p.att_mode = 2;
        st = run(3);
        p.att_mode = 0;
        if (st == SDK_OK) st = run(4);
        break;
      default: return SDK_ERR_INVALID_ARG;
    }
    if (st != SDK_OK) return st;
  }
  const cudaError_t last = cudaGetLastError();
  if (last != cudaSuccess && debug_launches())
    fprintf(stderr, "sdk: decode launches: %s\n", cudaGetErrorString(last));
  return last == cudaSuccess ? SDK_OK : SDK_ERR_CUDA;
}

}  // namespace sdk
