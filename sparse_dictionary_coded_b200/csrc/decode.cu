// Decode attention over dictionary codes with query-aware hierarchical
// sparsity ("LLM Inference in a Flash!", evolve.pub review, Summary: score
// all tokens with Klow=3 atoms, refine the top 10% with Khigh=16; FAQ on the
// 15x compression: only 3 atoms score most tokens).
//
// One layer, B sequences, R = B*Hq query heads.  Kernels, in stream order:
//   qd_kernel        QD[r][a] = <q_r, D_K[a]> (fp32 CUDA cores), and zeroes
//                    the per-head selection state, histograms and w.
//   klow_kernel      s_lo for every token from the 3 k_lo planes (12 B per
//                    token, coalesced) and QD staged in shared memory;
//                    writes order-preserving keys and the 12-bit radix
//                    histogram of every head.
//   pass2_kernel     finds the histogram bucket of the k-th key; tokens
//                    above it are selected, tokens inside it become
//                    candidates (compacted, with a second 12-bit histogram),
//                    tokens below go to the complement.
//   final_kernel     one CTA per head: last radix digit over the candidates,
//                    the exact k-th key, tie handling by token index, and
//                    the rest of the selected set.
//   rescore_kernel   s_t = scale * sum_{j<khigh} c_tj QD[idx_tj] for the
//                    selected tokens (64-byte k_full records).
//   value_kernel     p_t = exp(s_t - max) / z and the scatter
//                    w[idx^V_tj] += p_t c^V_tj (shared-memory fixed-point
//                    atomics into a per-atom weight tile per CTA; a cluster
//                    of CTAs per head sums its tiles through distributed
//                    shared memory).
//   out_kernel       out += w D_V over atom tiles (vector reductions into
//                    `out`, zeroed by qd_kernel).
#include <cooperative_groups.h>

#include "sdk_internal.cuh"

namespace sdk {


// Walk the flattened (head, entry) range [G0, G1).  Heads of sequence b have
// cnt[b] entries each; off[b] = sum_{b' < b} Hq * cnt[b'].  f(b, h, i0, i1)
// is called with block-uniform arguments.
template <class F>
__device__ __forceinline__ void for_segments(const int64_t* off, const int* cnt,
                                             int B, int64_t G0, int64_t G1,
                                             F f) {
  int64_t G = G0;
  int b = 0;
  while (G < G1) {
    while (b + 1 < B && off[b + 1] <= G) ++b;
    const int64_t local = G - off[b];
    const int c = cnt[b];
    const int h = (int)(local / c);
    const int64_t i = local - (int64_t)h * c;
    const int64_t take = min(G1 - G, (int64_t)c - i);
    f(b, h, i, i + take);
    G += take;
  }
}

// Block-wide search over NB histogram bins taken from the highest bin down:
// the bin holding the k-th element (1-based), the count in higher bins and
// the count in that bin.  s_tmp: >= 40 words of shared memory.  Sets
// *bad when k is 0 or exceeds the histogram total.
template <int NB>
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
    c[u] = rb < NB ? hist[NB - 1 - rb] : 0u;
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

// ---------------------------------------------------------------- qd_kernel
// QD[r][a] = sum_k q[r][k] D_K[a][k] on a 128-atom x 32-row tile.  The atom
// tile is kept as bf16 in shared memory ([k][atom]); thread (ta, tr) owns
// atoms 4ta..4ta+3 and rows 4tr..4tr+3 (16 accumulators, fp32 FMA chains in
// k order).  48 KB of shared memory per CTA lets four CTAs share an SM.
// The first kernel of a call also zeroes the per-head selection state, both
// histograms and `out` (accumulated with reductions by out_kernel).
constexpr int kQdThreads = 256;

template <int D>
__global__ void __launch_bounds__(kQdThreads) qd_kernel(DecodeParams p) {
  __shared__ __align__(16) uint16_t Ds[D][128];   // atom tile, k-major, bf16
  __shared__ __align__(16) float Qs[D][32];       // query rows, k-major
  const int n = p.n, R = p.R, tid = threadIdx.x;
  const int a0 = blockIdx.x * 128, r0 = blockIdx.y * 32;
  {
    const int64_t nthr = (int64_t)gridDim.x * gridDim.y * kQdThreads;
    const int64_t g0 = ((int64_t)blockIdx.y * gridDim.x + blockIdx.x) * kQdThreads + tid;
    const int64_t hwords = (int64_t)R * 4096;
    for (int64_t e = g0; e < hwords; e += nthr) {
      p.hist1[e] = 0u;
      p.hist2[e] = 0u;
    }
    for (int64_t e = g0; e < (int64_t)R * D; e += nthr) p.out[e] = 0.0f;
    for (int64_t e = g0; e < (int64_t)R; e += nthr) {
      sdk_select_state st;
      st.kth_key = 0u;
      st.k = (uint32_t)p.kcnt[e / p.Hq];
      st.n_above = st.n_cand = st.n_sel = st.n_comp = 0u;
      st.eq_total = st.eq_taken = 0u;
      st.max_score = 0u;
      st.max_comp = 0u;
      st.z = 0.0f;
#pragma unroll
      for (int u = 0; u < 5; ++u) st.pad[u] = 0u;
      p.st[e] = st;
    }
  }
  for (int e = tid; e < 128 * (D / 8); e += kQdThreads) {
    const int a = e & 127, c = e >> 7;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (a0 + a < n) v = __ldg(reinterpret_cast<const uint4*>(p.dk + (int64_t)(a0 + a) * D) + c);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      Ds[c * 8 + 2 * u][a] = (uint16_t)(w[u] & 0xFFFFu);
      Ds[c * 8 + 2 * u + 1][a] = (uint16_t)(w[u] >> 16);
    }
  }
  for (int e = tid; e < 32 * D; e += kQdThreads) {
    const int r = e & 31, k = e >> 5;
    Qs[k][r] = (r0 + r < R) ? __ldg(p.q + (int64_t)(r0 + r) * D + k) : 0.0f;
  }
  __syncthreads();
  const int ta = tid & 31, tr = tid >> 5;
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int u = 0; u < 4; ++u) acc[i][u] = 0.0f;
#pragma unroll 8
  for (int k = 0; k < D; ++k) {
    const uint2 dv = *reinterpret_cast<const uint2*>(&Ds[k][4 * ta]);
    const float4 qv = *reinterpret_cast<const float4*>(&Qs[k][4 * tr]);
    const float dd[4] = {bf16_lo(dv.x), bf16_hi(dv.x), bf16_lo(dv.y), bf16_hi(dv.y)};
    const float qq[4] = {qv.x, qv.y, qv.z, qv.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int u = 0; u < 4; ++u) acc[i][u] = fmaf(qq[i], dd[u], acc[i][u]);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = r0 + 4 * tr + i;
    if (r >= R) continue;
    float* dst = p.qd + (int64_t)r * n + a0 + 4 * ta;
    if (a0 + 4 * ta + 3 < n && (n & 3) == 0) {
      *reinterpret_cast<float4*>(dst) = make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
    } else {
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (a0 + 4 * ta + u < n) dst[u] = acc[i][u];
    }
  }
}

// Stage QD[r] (n floats) into shared memory.
__device__ __forceinline__ void stage_row(float* dst, const float* src, int n) {
  if ((n & 3) == 0 && ((reinterpret_cast<uintptr_t>(src) & 15) == 0)) {
    const float4* s4 = reinterpret_cast<const float4*>(src);
    float4* d4 = reinterpret_cast<float4*>(dst);
    for (int i = threadIdx.x; i < (n >> 2); i += blockDim.x) d4[i] = __ldg(s4 + i);
  } else {
    for (int i = threadIdx.x; i < n; i += blockDim.x) dst[i] = __ldg(src + i);
  }
}

// -------------------------------------------------------------- klow_kernel
constexpr int kScanThreads = 512;
constexpr int kKlowThreads = 1024;
constexpr int kKlowU = 4;   // tokens per thread per batch

__global__ void __launch_bounds__(kKlowThreads, 1) klow_kernel(DecodeParams p) {
  extern __shared__ float4 smem4[];
  float* sq = reinterpret_cast<float*>(smem4);
  uint32_t* sh = reinterpret_cast<uint32_t*>(sq + ((p.n + 3) & ~3));
  const int n = p.n, tid = threadIdx.x;
  const int64_t total = p.tok_off[p.B];
  const int64_t G0 = total * blockIdx.x / gridDim.x;
  const int64_t G1 = total * (blockIdx.x + 1) / gridDim.x;
  const int nlo = min(p.klow, kLoPlanes);

  for_segments(p.tok_off, p.lens, p.B, G0, G1, [&](int b, int h, int64_t t0, int64_t t1) {
    const int r = b * p.Hq + h, kvh = h / p.g;
    const float* qdr = p.qd + (int64_t)r * n;
    const bool stage = (t1 - t0) * p.klow >= (int64_t)(n / 2);
    if (stage) stage_row(sq, qdr, n);
    for (int i = tid; i < 4096; i += kKlowThreads) sh[i] = 0u;
    __syncthreads();
    const float* src = stage ? sq : qdr;
    const int64_t head = (int64_t)b * p.Hkv + kvh;
    const uint32_t* plane = p.k_lo + head * kLoPlanes * p.cap;
    const uint32_t* rec = p.k_full + head * p.cap * kAtoms;
    uint32_t* keys = p.keys + (int64_t)r * p.L;
    constexpr int64_t kBatch = (int64_t)kKlowU * kKlowThreads;
    // register double buffer: the next batch's plane words are in flight
    // while the current batch is scored
    uint32_t wv[kKlowU][kLoPlanes], wn[kKlowU][kLoPlanes];
    auto load_batch = [&](int64_t tb, uint32_t (&w)[kKlowU][kLoPlanes]) {
#pragma unroll
      for (int u = 0; u < kKlowU; ++u) {
        const int64_t t = tb + tid + u * kKlowThreads;
#pragma unroll
        for (int j = 0; j < kLoPlanes; ++j)
          w[u][j] = (t < t1 && j < nlo) ? __ldcs(plane + j * p.cap + t) : 0u;
      }
    };
    load_batch(t0, wv);
    for (int64_t tb = t0; tb < t1; tb += kBatch) {
      if (tb + kBatch < t1) load_batch(tb + kBatch, wn);
#pragma unroll
      for (int u = 0; u < kKlowU; ++u) {
        const int64_t t = tb + tid + u * kKlowThreads;
        if (t >= t1) continue;
        float s = 0.0f;
#pragma unroll
        for (int j = 0; j < kLoPlanes; ++j) {
          if (j >= nlo) break;
          const uint32_t idx = word_idx(wv[u][j]);
          if (idx >= (uint32_t)n) {
            record_error(p.hdr, SDK_ERR_DEVICE_CHECK, idx);
            continue;
          }
          s = fmaf(word_coef(wv[u][j]), src[idx], s);
        }
        for (int j = kLoPlanes; j < p.klow; ++j) {
          const uint32_t wj = __ldg(rec + t * kAtoms + j);
          const uint32_t idx = word_idx(wj);
          if (idx >= (uint32_t)n) {
            record_error(p.hdr, SDK_ERR_DEVICE_CHECK, idx);
            continue;
          }
          s = fmaf(word_coef(wj), src[idx], s);
        }
        const uint32_t key = score_key(s);
        keys[t] = key;
        atomicAdd(&sh[key >> 20], 1u);
      }
#pragma unroll
      for (int u = 0; u < kKlowU; ++u)
#pragma unroll
        for (int j = 0; j < kLoPlanes; ++j) wv[u][j] = wn[u][j];
    }
    __syncthreads();
    uint32_t* gh = p.hist1 + (int64_t)r * 4096;
    for (int i = tid; i < 4096; i += kKlowThreads)
      if (sh[i]) atomicAdd(&gh[i], sh[i]);
    __syncthreads();
  });
}

// ------------------------------------------------------------- pass2_kernel
// Tokens above the bucket of the k-th key are selected, tokens inside it
// become candidates (with a histogram of key bits 19..8), the others go to
// the complement.  Each warp compacts 128 tokens per iteration with ballots
// and reserves its output slots with one atomic per category.
__global__ void __launch_bounds__(kScanThreads, 2) pass2_kernel(DecodeParams p) {
  __shared__ uint32_t s_tmp[48];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const unsigned lt = (1u << lane) - 1u;
  const int64_t total = p.tok_off[p.B];
  const int64_t G0 = total * blockIdx.x / gridDim.x;
  const int64_t G1 = total * (blockIdx.x + 1) / gridDim.x;

  for_segments(p.tok_off, p.lens, p.B, G0, G1, [&](int b, int h, int64_t t0, int64_t t1) {
    const int r = b * p.Hq + h;
    const int Nb = p.lens[b];
    sdk_select_state* st = p.st + r;
    uint32_t b1, above1, cnt1;
    bool bad;
    block_find_desc<4096>(p.hist1 + (int64_t)r * 4096, (uint32_t)p.kcnt[b], s_tmp, b1, above1,
                          cnt1, bad);
    if (bad) {
      if (tid == 0) record_error(p.hdr, SDK_ERR_DEVICE_CHECK, 0x10000000u | r);
      return;
    }
    if (t0 == 0 && tid == 0) st->n_above = above1;
    const uint32_t* keys = p.keys + (int64_t)r * p.L;
    int32_t* list = p.list + (int64_t)r * p.L;
    int32_t* ct = p.cand_t + (int64_t)r * p.L;
    uint32_t* ck = p.cand_key + (int64_t)r * p.L;
    uint32_t* h2 = p.hist2 + (int64_t)r * 4096;
    uint32_t cmax = 0u;
    const int nwarps = kScanThreads / 32;
    constexpr int U = 4;                       // tokens per lane per batch
    constexpr int64_t WB = 32 * U;             // tokens per warp batch
    uint32_t kc[U], kn[U];
    auto load_keys = [&](int64_t tb, uint32_t (&kk)[U]) {
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int64_t t = tb + lane + 32 * u;
        kk[u] = t < t1 ? keys[t] : 0u;
      }
    };
    int64_t tb = t0 + (int64_t)warp * WB;
    if (tb < t1) load_keys(tb, kc);
    for (; tb < t1; tb += (int64_t)nwarps * WB) {
      const int64_t tnext = tb + (int64_t)nwarps * WB;
      if (tnext < t1) load_keys(tnext, kn);
      unsigned ms[U], mc[U], mo[U];
      uint32_t ns = 0, nc = 0, no = 0;
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const bool valid = tb + lane + 32 * u < t1;
        const uint32_t d1 = kc[u] >> 20;
        ms[u] = __ballot_sync(0xffffffffu, valid && d1 > b1);
        mc[u] = __ballot_sync(0xffffffffu, valid && d1 == b1);
        mo[u] = __ballot_sync(0xffffffffu, valid && d1 < b1 && p.full);
        ns += __popc(ms[u]);
        nc += __popc(mc[u]);
        no += __popc(mo[u]);
      }
      uint32_t bs = 0, bc = 0, bo = 0;
      if (lane == 0) {
        if (ns) bs = atomicAdd(&st->n_sel, ns);
        if (nc) bc = atomicAdd(&st->n_cand, nc);
        if (no) bo = atomicAdd(&st->n_comp, no);
      }
      bs = __shfl_sync(0xffffffffu, bs, 0);
      bc = __shfl_sync(0xffffffffu, bc, 0);
      bo = __shfl_sync(0xffffffffu, bo, 0);
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int64_t t = tb + lane + 32 * u;
        if ((ms[u] >> lane) & 1u) {
          const uint32_t pos = bs + __popc(ms[u] & lt);
          if (pos < (uint32_t)Nb) list[pos] = (int32_t)t;
        } else if ((mc[u] >> lane) & 1u) {
          const uint32_t pos = bc + __popc(mc[u] & lt);
          if (pos < (uint32_t)Nb) {
            ct[pos] = (int32_t)t;
            ck[pos] = kc[u];
          }
          atomicAdd(&h2[(kc[u] >> 8) & 0xFFFu], 1u);
        } else if ((mo[u] >> lane) & 1u) {
          const uint32_t pos = bo + __popc(mo[u] & lt);
          if (pos < (uint32_t)Nb) list[Nb - 1 - (int64_t)pos] = (int32_t)t;
          cmax = max(cmax, kc[u]);
        }
        bs += __popc(ms[u]);
        bc += __popc(mc[u]);
        bo += __popc(mo[u]);
      }
#pragma unroll
      for (int u = 0; u < U; ++u) kc[u] = kn[u];
    }
    if (p.full) {
      cmax = warp_umax(cmax);
      if (lane == 0 && cmax) atomicMax(&st->max_comp, cmax);
    }
    __syncthreads();
  });
}

// ------------------------------------------------------------- final_kernel
constexpr int kFinalStage = 12288;   // candidates staged in shared memory
// One CTA per query head: the last two radix digits over the candidates, the
// exact k-th key, the tie rule (lower token index first) and the rest of the
// selected set.
__global__ void __launch_bounds__(kScanThreads) final_kernel(DecodeParams p) {
  __shared__ uint32_t s_tmp[48];
  __shared__ uint32_t sh[2048];
  __shared__ uint32_t s_cnt[2];
  const int r = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const unsigned lt = (1u << lane) - 1u;
  const int b = r / p.Hq;
  const int Nb = p.lens[b];
  const uint32_t k = (uint32_t)p.kcnt[b];
  sdk_select_state* st = p.st + r;
  const uint32_t n_cand = st->n_cand;
  const uint32_t n_above = st->n_above;
  if (st->n_sel != n_above || n_above >= k || n_cand == 0u || n_cand > (uint32_t)Nb) {
    if (tid == 0) record_error(p.hdr, SDK_ERR_DEVICE_CHECK, 0x20000000u | r);
    return;
  }
  const uint32_t* ck = p.cand_key + (int64_t)r * p.L;
  const int32_t* ct = p.cand_t + (int64_t)r * p.L;
  int32_t* list = p.list + (int64_t)r * p.L;
  const uint32_t k1 = k - n_above;
  // candidates in shared memory when they fit (one coalesced pass over the
  // global copy; the passes below then read shared memory)
  extern __shared__ uint32_t s_cand[];
  if (n_cand <= (uint32_t)kFinalStage) {
    for (uint32_t i = tid; i < n_cand; i += kScanThreads) {
      s_cand[i] = ck[i];
      s_cand[kFinalStage + i] = (uint32_t)ct[i];
    }
    __syncthreads();
    ck = s_cand;
    ct = reinterpret_cast<const int32_t*>(s_cand + kFinalStage);
  }

  uint32_t b2, above2, cnt2, b3, above3, cnt3;
  bool bad;
  block_find_desc<4096>(p.hist2 + (int64_t)r * 4096, k1, s_tmp, b2, above2, cnt2, bad);
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
  // ties, by radix select over index digits 31..21, 20..10, 9..0 (bins kept
  // in reverse so the descending search walks ascending indices)
  uint32_t t_cut = 0xFFFFFFFFu;
  if (eq_total > eq_take) {
    uint32_t prefix = 0u, rank = eq_take;
    for (int ps = 0; ps < 3; ++ps) {
      const int sh_lo = ps == 0 ? 21 : (ps == 1 ? 10 : 0);
      const int wbits = ps == 2 ? 10 : 11;
      const uint32_t nb = 1u << wbits;
      for (int i = tid; i < 2048; i += kScanThreads) sh[i] = 0u;
      __syncthreads();
      for (uint32_t i = tid; i < n_cand; i += kScanThreads) {
        if (ck[i] != T) continue;
        const uint32_t t = (uint32_t)ct[i];
        const uint32_t hi = (ps == 0) ? 0u : (t >> (sh_lo + wbits));
        if (hi != prefix) continue;
        atomicAdd(&sh[2047u - ((t >> sh_lo) & (nb - 1u))], 1u);
      }
      __syncthreads();
      uint32_t bin, above, cnt;
      block_find_desc<2048>(sh, rank, s_tmp, bin, above, cnt, bad);
      if (bad) {
        if (tid == 0) record_error(p.hdr, SDK_ERR_DEVICE_CHECK, 0x23000000u | r);
        return;
      }
      prefix = (prefix << wbits) | (2047u - bin);
      rank -= above;
    }
    t_cut = prefix;
  }

  if (tid == 0) {
    s_cnt[0] = n_above;
    s_cnt[1] = st->n_comp;
  }
  __syncthreads();
  uint32_t cmax = 0u;
  for (uint32_t i0 = (uint32_t)warp * 32; i0 < n_cand; i0 += kScanThreads) {
    const uint32_t i = i0 + lane;
    uint32_t key = 0u, t = 0u;
    bool sel = false, comp = false;
    if (i < n_cand) {
      key = ck[i];
      t = (uint32_t)ct[i];
      sel = key > T || (key == T && t <= t_cut);
      comp = !sel && p.full;
    }
    const unsigned msel = __ballot_sync(0xffffffffu, sel);
    const unsigned mcomp = __ballot_sync(0xffffffffu, comp);
    uint32_t bs = 0, bo = 0;
    if (lane == 0) {
      if (msel) bs = atomicAdd(&s_cnt[0], (uint32_t)__popc(msel));
      if (mcomp) bo = atomicAdd(&s_cnt[1], (uint32_t)__popc(mcomp));
    }
    bs = __shfl_sync(0xffffffffu, bs, 0) + __popc(msel & lt);
    bo = __shfl_sync(0xffffffffu, bo, 0) + __popc(mcomp & lt);
    if (sel) {
      if (bs < k) list[bs] = (int32_t)t;
      else record_error(p.hdr, SDK_ERR_DEVICE_CHECK, 0x26000000u | r);
    }
    if (comp) {
      if (bo < (uint32_t)Nb) list[Nb - 1 - (int64_t)bo] = (int32_t)t;
      else record_error(p.hdr, SDK_ERR_DEVICE_CHECK, 0x27000000u | r);
      cmax = max(cmax, key);
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

// ----------------------------------------------------------- rescore_kernel
// s_t = scale * sum_{j<khigh} c_tj QD[idx_tj] for the selected tokens.  Four
// lanes share a token: lane c of the group loads words 4c..4c+3 of the
// 64-byte record (one coalesced 16-byte load; the group reads the record in
// full), gathers their QD terms and the group sums its partials with two
// shuffles.  A ring of kRing iterations keeps list entries and records in
// flight ahead of the one being scored.
constexpr int kRecThreads = 1024;
constexpr int kRing = 4;

__global__ void __launch_bounds__(kRecThreads, 1) rescore_kernel(DecodeParams p) {
  extern __shared__ float4 smem4[];
  float* sq = reinterpret_cast<float*>(smem4);
  const int n = p.n, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int grp = lane >> 2, c = lane & 3;
  constexpr int kWarps = kRecThreads / 32;
  const int64_t total = p.sel_off[p.B];
  const int64_t G0 = total * blockIdx.x / gridDim.x;
  const int64_t G1 = total * (blockIdx.x + 1) / gridDim.x;

  for_segments(p.sel_off, p.kcnt, p.B, G0, G1, [&](int b, int h, int64_t i0, int64_t i1) {
    const int r = b * p.Hq + h, kvh = h / p.g;
    const float* qdr = p.qd + (int64_t)r * n;
    const bool stage = (i1 - i0) * p.khigh >= (int64_t)(n / 2);
    if (stage) stage_row(sq, qdr, n);
    __syncthreads();
    const float* src = stage ? sq : qdr;
    const uint4* rec = reinterpret_cast<const uint4*>(p.k_full +
                                                      ((int64_t)b * p.Hkv + kvh) * p.cap * kAtoms);
    const int32_t* list = p.list + (int64_t)r * p.L;
    float* out = p.sel_score + (int64_t)r * p.L;
    const int Nb = p.lens[b];
    const int jmax = min(p.khigh - 4 * c, 4);   // words of this lane that count
    auto entry = [&](int64_t it) { return i0 + (it * kWarps + warp) * 8 + grp; };
    auto fetch = [&](int64_t it, int& t, uint4& w) {
      const int64_t i = entry(it);
      t = i < i1 ? list[i] : -1;
      if (i < i1 && (t < 0 || t >= Nb)) {
        if (c == 0) record_error(p.hdr, SDK_ERR_DEVICE_CHECK, 0x30000000u | r);
        t = -1;
      }
      w = t >= 0 ? __ldcs(rec + (int64_t)t * 4 + c) : make_uint4(0u, 0u, 0u, 0u);
    };
    int tq[kRing];
    uint4 wq[kRing];
#pragma unroll
    for (int s2 = 0; s2 < kRing; ++s2) fetch(s2, tq[s2], wq[s2]);
    float smax = -INFINITY;
    for (int64_t it0 = 0; entry(it0) - grp < i1; it0 += kRing) {
#pragma unroll
      for (int s2 = 0; s2 < kRing; ++s2) {
        const int64_t it = it0 + s2;
        const int64_t i = entry(it);
        const int t = tq[s2];
        const uint4 w = wq[s2];
        fetch(it + kRing, tq[s2], wq[s2]);
        const uint32_t wd[4] = {w.x, w.y, w.z, w.w};
        float part = 0.0f;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          if (u >= jmax) break;
          const uint32_t idx = word_idx(wd[u]);
          if (t >= 0 && idx >= (uint32_t)n) {
            record_error(p.hdr, SDK_ERR_DEVICE_CHECK, idx);
            continue;
          }
          if (t >= 0) part = fmaf(word_coef(wd[u]), src[idx], part);
        }
        part += __shfl_xor_sync(0xffffffffu, part, 1);
        part += __shfl_xor_sync(0xffffffffu, part, 2);
        if (c == 0 && i < i1) {
          const float sc = t >= 0 ? part * p.scale : -INFINITY;
          out[i] = sc;
          smax = fmaxf(smax, sc);
        }
      }
    }
    smax = warp_max(smax);
    if (lane == 0 && smax > -INFINITY) atomicMax(&p.st[r].max_score, score_key(smax));
    __syncthreads();
  });
}

// ------------------------------------------------------------- value_kernel
// One cluster of C CTAs per query head; CTA `rank` owns a contiguous share
// of the head's softmax domain (the selected set, or every token with the
// full-softmax flag).
//   pass A  e_t = exp(logit_t - max); the cluster sums e_t into z
//           (distributed shared memory).
//   pass B  p_t = e_t / z; w[idx^V_tj] += p_t c^V_tj into a shared-memory
//           tile of n bins, four lanes per token as in rescore_kernel.  The
//           bins hold 2^-20 fixed point in int32 (native shared-memory
//           integer atomics, exact and order-independent).  Since
//           sum_t p_t = 1, a bin can leave the int32 range only if the
//           CTA's sum of |p_t c_tj| reaches 2^10; a CTA that sees that
//           re-runs pass B with fp32 atomics.
//   reduce  each CTA sums its slice of the atoms over the cluster's tiles
//           and writes w[r] (already normalised) with plain stores.
constexpr float kFixScale = 1048576.0f;       // 2^20
constexpr float kFixInv = 1.0f / 1048576.0f;

__global__ void __launch_bounds__(kRecThreads, 1) value_kernel(DecodeParams p, int C) {
  extern __shared__ float4 smem4[];
  int* siw = reinterpret_cast<int*>(smem4);
  float* sfw = reinterpret_cast<float*>(smem4);
  __shared__ float s_red[kRecThreads / 32];
  __shared__ float s_z;
  __shared__ int s_float;
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  const int n = p.n, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int grp = lane >> 2, c = lane & 3;
  constexpr int kWarps = kRecThreads / 32;
  const int r = blockIdx.x / C;
  const int rank = (int)cluster.block_rank();
  const int b = r / p.Hq, h = r % p.Hq, kvh = h / p.g;
  const int64_t Dr = p.dcnt[b];
  const int64_t i0 = Dr * rank / C, i1 = Dr * (rank + 1) / C;
  const int k = p.kcnt[b];
  const int Nb = p.lens[b];
  const sdk_select_state* st = p.st + r;
  float m = key_score(st->max_score);
  if (p.full && st->n_comp > 0u) m = fmaxf(m, p.scale * key_score(st->max_comp));
  const uint4* rec = reinterpret_cast<const uint4*>(p.v_full +
                                                    ((int64_t)b * p.Hkv + kvh) * p.cap * kAtoms);
  const int32_t* list = p.list + (int64_t)r * p.L;
  const float* ss = p.sel_score + (int64_t)r * p.L;
  const uint32_t* keys = p.keys + (int64_t)r * p.L;
  auto logit_of = [&](int64_t i, int64_t t) {
    return (i < k) ? ss[i] : p.scale * key_score(keys[t]);
  };

  for (int i = tid; i < n; i += kRecThreads) siw[i] = 0;
  // ---- pass A: z
  float z = 0.0f;
  for (int64_t i = i0 + tid; i < i1; i += kRecThreads) {
    const int64_t t = i < k ? 0 : (int64_t)list[i];
    if (t < 0 || t >= Nb) continue;
    z += expf(logit_of(i, t) - m);
  }
  z = warp_sum(z);
  if (lane == 0) s_red[warp] = z;
  __syncthreads();
  if (tid == 0) {
    float zz = 0.0f;
    for (int i = 0; i < kWarps; ++i) zz += s_red[i];
    s_z = zz;
    s_float = 0;
  }
  cluster.sync();
  float ztot = 0.0f;
  for (int cc = 0; cc < C; ++cc) ztot += *cluster.map_shared_rank(&s_z, cc);
  const float invz = 1.0f / ztot;

  // ---- pass B: scatter p_t c_tj (fixed point; fp32 atomics on re-run)
  auto entry = [&](int64_t it) { return i0 + (it * kWarps + warp) * 8 + grp; };
  auto fetch = [&](int64_t it, int& t, uint4& w) {
    const int64_t i = entry(it);
    t = i < i1 ? list[i] : -1;
    if (i < i1 && (t < 0 || t >= Nb)) {
      if (c == 0) record_error(p.hdr, SDK_ERR_DEVICE_CHECK, 0x31000000u | r);
      t = -1;
    }
    w = t >= 0 ? __ldcs(rec + (int64_t)t * 4 + c) : make_uint4(0u, 0u, 0u, 0u);
  };
  for (int pass = 0; pass < 2; ++pass) {
    const bool use_float = pass == 1;
    if (use_float) {
      if (!s_float) break;
      __syncthreads();
      for (int i = tid; i < n; i += kRecThreads) sfw[i] = 0.0f;
    }
    __syncthreads();
    float absum = 0.0f;
    int tq[kRing];
    uint4 wq[kRing];
#pragma unroll
    for (int s2 = 0; s2 < kRing; ++s2) fetch(s2, tq[s2], wq[s2]);
    for (int64_t it0 = 0; entry(it0) - grp < i1; it0 += kRing) {
#pragma unroll
      for (int s2 = 0; s2 < kRing; ++s2) {
        const int64_t it = it0 + s2;
        const int64_t i = entry(it);
        const int t = tq[s2];
        const uint4 w = wq[s2];
        fetch(it + kRing, tq[s2], wq[s2]);
        if (t < 0) continue;
        const float pt = expf(logit_of(i, t) - m) * invz;
        const uint32_t wd[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const uint32_t idx = word_idx(wd[u]);
          if (idx >= (uint32_t)n) {
            record_error(p.hdr, SDK_ERR_DEVICE_CHECK, idx);
            continue;
          }
          const float v = pt * word_coef(wd[u]);
          if (use_float) {
            atomicAdd(&sfw[idx], v);
          } else {
            absum += fabsf(v);
            atomicAdd(&siw[idx], __float2int_rn(v * kFixScale));
          }
        }
      }
    }
    if (!use_float) {
      // exact int32 range guard (see above); also catches NaN
      if (!(absum < 1024.0f)) s_float = 1;
      __syncthreads();
      if (s_float) continue;
      break;
    }
  }
  cluster.sync();
  // reduce this CTA's slice of the atoms over the C tiles of the cluster
  const int a0 = (int)((int64_t)n * rank / C), a1 = (int)((int64_t)n * (rank + 1) / C);
  float* gw = p.w + (int64_t)r * n;
  for (int a = a0 + tid; a < a1; a += kRecThreads) {
    float sum = 0.0f;
    for (int cc = 0; cc < C; ++cc) {
      const bool f = *cluster.map_shared_rank(&s_float, cc) != 0;
      const int* tile = cluster.map_shared_rank(siw, cc);
      sum += f ? __int_as_float(tile[a]) : (float)tile[a] * kFixInv;
    }
    gw[a] = sum;
  }
  if (rank == 0 && tid == 0) p.st[r].z = ztot;
  cluster.sync();
}

// --------------------------------------------------------------- out_kernel
// out[r][k] += sum_{a in tile} w[r][a] D_V[a][k] over a 128-atom tile and a
// 32-row block.  The atom tile stays bf16 in shared memory ([atom][k]);
// thread (tk, tr) owns columns tk*C.. and rows 4tr..4tr+3; results are
// added with vector reductions into `out` (zeroed by qd_kernel).
template <int D>
__global__ void __launch_bounds__(kQdThreads) out_kernel(DecodeParams p) {
  __shared__ __align__(16) uint16_t Ds[128][D];   // atom tile, bf16
  __shared__ __align__(16) float Ws[128][32];     // w tile, [atom][row]
  const int n = p.n, R = p.R, tid = threadIdx.x;
  const int a0 = blockIdx.x * 128, r0 = blockIdx.y * 32;
  for (int e = tid; e < 128 * (D / 8); e += kQdThreads) {
    const int a = e / (D / 8), c = e % (D / 8);
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (a0 + a < n) v = __ldg(reinterpret_cast<const uint4*>(p.dv + (int64_t)(a0 + a) * D) + c);
    *reinterpret_cast<uint4*>(&Ds[a][c * 8]) = v;
  }
  for (int e = tid; e < 128 * 32; e += kQdThreads) {
    const int r = e & 31, a = e >> 5;
    Ws[a][r] = (r0 + r < R && a0 + a < n) ? p.w[(int64_t)(r0 + r) * n + a0 + a] : 0.0f;
  }
  __syncthreads();
  constexpr int C = D / 32;
  const int tk = tid & 31, tr = tid >> 5;
  float acc[4][C];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int cc = 0; cc < C; ++cc) acc[i][cc] = 0.0f;
#pragma unroll 8
  for (int a = 0; a < 128; ++a) {
    float dv[C];
    if constexpr (C == 4) {
      const uint2 v = *reinterpret_cast<const uint2*>(&Ds[a][tk * 4]);
      dv[0] = bf16_lo(v.x); dv[1] = bf16_hi(v.x); dv[2] = bf16_lo(v.y); dv[3] = bf16_hi(v.y);
    } else {
      const uint32_t v = *reinterpret_cast<const uint32_t*>(&Ds[a][tk * 2]);
      dv[0] = bf16_lo(v); dv[1] = bf16_hi(v);
    }
    const float4 wv = *reinterpret_cast<const float4*>(&Ws[a][4 * tr]);
    const float wr[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int cc = 0; cc < C; ++cc) acc[i][cc] = fmaf(wr[i], dv[cc], acc[i][cc]);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = r0 + 4 * tr + i;
    if (r >= R) continue;
    float* dst = p.out + (int64_t)r * D + tk * C;
    if constexpr (C == 4) {
      asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(dst), "f"(acc[i][0]),
                   "f"(acc[i][1]), "f"(acc[i][2]), "f"(acc[i][3])
                   : "memory");
    } else {
      asm volatile("red.global.add.v2.f32 [%0], {%1, %2};" ::"l"(dst), "f"(acc[i][0]),
                   "f"(acc[i][1])
                   : "memory");
    }
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
  l.w = take(R * n * 4);
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

sdk_status launch_decode(const DecodeParams& p, cudaStream_t stream) {
  const int sms = num_sms();
  const size_t qd_smem = (size_t)((p.n + 3) & ~3) * 4;
  static bool attr = false;
  if (!attr) {
    cudaFuncSetAttribute(klow_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
    cudaFuncSetAttribute(rescore_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
    cudaFuncSetAttribute(final_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
    cudaFuncSetAttribute(value_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
    cudaFuncSetAttribute(value_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 0);
    attr = true;
  }
  {
    dim3 grid((p.n + 127) / 128, (p.R + 31) / 32);
    if (p.d == 128) qd_kernel<128><<<grid, kQdThreads, 0, stream>>>(p);
    else qd_kernel<64><<<grid, kQdThreads, 0, stream>>>(p);
  }
  {
    const int g = grid_for(p.tok_off[p.B], 2048, sms);
    klow_kernel<<<g, kKlowThreads, qd_smem + 4096 * 4, stream>>>(p);
  }
  {
    const int g = grid_for(p.tok_off[p.B], 8192, 2 * sms);
    pass2_kernel<<<g, kScanThreads, 0, stream>>>(p);
  }
  final_kernel<<<p.R, kScanThreads, (size_t)2 * kFinalStage * 4, stream>>>(p);
  {
    int64_t per = p.sel_off[p.B] / sms;
    if (per < 1024) per = 1024;
    const int g = grid_for(p.sel_off[p.B], per, sms);
    rescore_kernel<<<g, kRecThreads, qd_smem, stream>>>(p);
  }
  {
    int64_t dmax = 0;
    for (int b = 0; b < p.B; ++b) dmax = p.dcnt[b] > dmax ? p.dcnt[b] : dmax;
    int C = 1;
    while (C < 8 && (int64_t)p.R * C * 2 <= sms && dmax / (2 * C) >= 1024) C *= 2;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(p.R * C));
    cfg.blockDim = dim3(kRecThreads);
    cfg.dynamicSmemBytes = qd_smem;
    cfg.stream = stream;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = (unsigned)C;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, value_kernel, p, C) != cudaSuccess) return SDK_ERR_CUDA;
  }
  {
    dim3 grid((p.n + 127) / 128, (p.R + 31) / 32);
    if (p.d == 128) out_kernel<128><<<grid, kQdThreads, 0, stream>>>(p);
    else out_kernel<64><<<grid, kQdThreads, 0, stream>>>(p);
  }
  return cudaGetLastError() == cudaSuccess ? SDK_OK : SDK_ERR_CUDA;
}

}  // namespace sdk
