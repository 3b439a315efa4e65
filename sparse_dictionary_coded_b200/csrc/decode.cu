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
//   value_kernel     e_t = exp(s_t - max), z = sum e_t, and the scatter
//                    w[idx^V_tj] += e_t c^V_tj (shared-memory atomics into a
//                    per-atom weight tile, flushed to global).
//   out_kernel       partial sums of w D_V over atom tiles;
//   out_reduce       out = (sum of partials) / z.
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
template <int D>
__global__ void __launch_bounds__(256) qd_kernel(DecodeParams p) {
  __shared__ float Ds[D][64];
  __shared__ float Qs[D][32];
  const int n = p.n, R = p.R;
  const int a0 = blockIdx.x * 64, r0 = blockIdx.y * 32;
  const int tid = threadIdx.x;

  // zero the per-head selection state and histograms (grid-stride over the
  // whole grid, block-linear order)
  {
    const int64_t nblk = (int64_t)gridDim.x * gridDim.y;
    const int64_t bl = (int64_t)blockIdx.y * gridDim.x + blockIdx.x;
    const int64_t hwords = (int64_t)R * 4096;
    for (int64_t e = bl * 256 + tid; e < hwords; e += nblk * 256) {
      p.hist1[e] = 0u;
      p.hist2[e] = 0u;
    }
    for (int64_t e = bl * 256 + tid; e < (int64_t)R; e += nblk * 256) {
      sdk_select_state s;
      const int b = (int)(e / p.Hq);
      s.kth_key = 0u;
      s.k = (uint32_t)p.kcnt[b];
      s.n_above = s.n_cand = s.n_sel = s.n_comp = 0u;
      s.eq_total = s.eq_taken = 0u;
      s.max_score = 0u;
      s.max_comp = 0u;
      s.z = 0.0f;
#pragma unroll
      for (int u = 0; u < 5; ++u) s.pad[u] = 0u;
      p.st[e] = s;
    }
  }

  // atom tile, transposed to [k][a] in fp32
  for (int e = tid; e < 64 * (D / 8); e += 256) {
    const int a = e & 63, c = e >> 6;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (a0 + a < n)
      v = __ldg(reinterpret_cast<const uint4*>(p.dk + (int64_t)(a0 + a) * D) + c);
    Ds[c * 8 + 0][a] = bf16_lo(v.x);
    Ds[c * 8 + 1][a] = bf16_hi(v.x);
    Ds[c * 8 + 2][a] = bf16_lo(v.y);
    Ds[c * 8 + 3][a] = bf16_hi(v.y);
    Ds[c * 8 + 4][a] = bf16_lo(v.z);
    Ds[c * 8 + 5][a] = bf16_hi(v.z);
    Ds[c * 8 + 6][a] = bf16_lo(v.w);
    Ds[c * 8 + 7][a] = bf16_hi(v.w);
  }
  for (int e = tid; e < 32 * D; e += 256) {
    const int r = e & 31, k = e >> 5;
    Qs[k][r] = (r0 + r < R) ? p.q[(int64_t)(r0 + r) * D + k] : 0.0f;
  }
  __syncthreads();

  const int ta = tid & 31, tr = tid >> 5;
  float acc[4][2];
#pragma unroll
  for (int i = 0; i < 4; ++i) acc[i][0] = acc[i][1] = 0.0f;
#pragma unroll 8
  for (int k = 0; k < D; ++k) {
    const float2 dv = *reinterpret_cast<const float2*>(&Ds[k][2 * ta]);
    const float4 qv = *reinterpret_cast<const float4*>(&Qs[k][4 * tr]);
    acc[0][0] = fmaf(qv.x, dv.x, acc[0][0]);
    acc[0][1] = fmaf(qv.x, dv.y, acc[0][1]);
    acc[1][0] = fmaf(qv.y, dv.x, acc[1][0]);
    acc[1][1] = fmaf(qv.y, dv.y, acc[1][1]);
    acc[2][0] = fmaf(qv.z, dv.x, acc[2][0]);
    acc[2][1] = fmaf(qv.z, dv.y, acc[2][1]);
    acc[3][0] = fmaf(qv.w, dv.x, acc[3][0]);
    acc[3][1] = fmaf(qv.w, dv.y, acc[3][1]);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = r0 + 4 * tr + i;
    if (r >= R) continue;
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int a = a0 + 2 * ta + u;
      if (a < n) {
        p.qd[(int64_t)r * n + a] = acc[i][u];
        p.w[(int64_t)r * n + a] = 0.0f;
      }
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

__global__ void __launch_bounds__(kScanThreads, 1) klow_kernel(DecodeParams p) {
  extern __shared__ float4 smem4[];
  float* sq = reinterpret_cast<float*>(smem4);
  uint32_t* sh = reinterpret_cast<uint32_t*>(sq + ((p.n + 3) & ~3));
  const int n = p.n, tid = threadIdx.x;
  const int64_t total = p.tok_off[p.B];
  const int64_t G0 = total * blockIdx.x / gridDim.x;
  const int64_t G1 = total * (blockIdx.x + 1) / gridDim.x;
  const int nlo = min(p.klow, kLoPlanes);

  for_segments(p.tok_off, p.lens, p.B, G0, G1,
               [&](int b, int h, int64_t t0, int64_t t1) {
    const int r = b * p.Hq + h, kvh = h / p.g;
    const float* qdr = p.qd + (int64_t)r * n;
    const bool stage = (t1 - t0) * p.klow >= (int64_t)(n / 2);
    if (stage) stage_row(sq, qdr, n);
    for (int i = tid; i < 4096; i += kScanThreads) sh[i] = 0u;
    __syncthreads();
    const float* src = stage ? sq : qdr;
    const int64_t head = (int64_t)b * p.Hkv + kvh;
    const uint32_t* plane = p.k_lo + head * kLoPlanes * p.cap;
    const uint32_t* rec = p.k_full + head * p.cap * kAtoms;
    uint32_t* keys = p.keys + (int64_t)r * p.L;
    for (int64_t tb = t0; tb < t1; tb += 4 * kScanThreads) {
      uint32_t wv[4][kLoPlanes];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int64_t t = tb + tid + u * kScanThreads;
#pragma unroll
        for (int j = 0; j < kLoPlanes; ++j)
          wv[u][j] = (t < t1 && j < nlo) ? __ldcs(plane + j * p.cap + t) : 0u;
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int64_t t = tb + tid + u * kScanThreads;
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
    }
    __syncthreads();
    uint32_t* gh = p.hist1 + (int64_t)r * 4096;
    for (int i = tid; i < 4096; i += kScanThreads)
      if (sh[i]) atomicAdd(&gh[i], sh[i]);
    __syncthreads();
  });
}

// ------------------------------------------------------------- pass2_kernel
constexpr int kPass2PerThread = 4;

__global__ void __launch_bounds__(kScanThreads) pass2_kernel(DecodeParams p) {
  __shared__ uint32_t s_tmp[48];
  __shared__ uint32_t s_base[4];
  const int tid = threadIdx.x;
  const int64_t total = p.tok_off[p.B];
  const int64_t G0 = total * blockIdx.x / gridDim.x;
  const int64_t G1 = total * (blockIdx.x + 1) / gridDim.x;

  for_segments(p.tok_off, p.lens, p.B, G0, G1,
               [&](int b, int h, int64_t t0, int64_t t1) {
    const int r = b * p.Hq + h;
    const int Nb = p.lens[b];
    sdk_select_state* st = p.st + r;
    uint32_t b1, above1, cnt1;
    bool bad;
    block_find_desc<4096>(p.hist1 + (int64_t)r * 4096, (uint32_t)p.kcnt[b],
                          s_tmp, b1, above1, cnt1, bad);
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
    for (int64_t tb = t0; tb < t1; tb += kPass2PerThread * kScanThreads) {
      uint32_t key[kPass2PerThread];
      uint32_t nsel = 0, ncand = 0, ncomp = 0;
#pragma unroll
      for (int u = 0; u < kPass2PerThread; ++u) {
        const int64_t t = tb + tid + u * kScanThreads;
        key[u] = t < t1 ? keys[t] : 0u;
        if (t < t1) {
          const uint32_t d1 = key[u] >> 20;
          if (d1 > b1) ++nsel;
          else if (d1 == b1) ++ncand;
          else ++ncomp;
        }
      }
      uint32_t tot_sc, tot_comp;
      const uint32_t inc_sc = block_incl_scan(nsel | (ncand << 16), s_tmp, &tot_sc);
      const uint32_t inc_comp = p.full ? block_incl_scan(ncomp, s_tmp, &tot_comp) : 0u;
      if (tid == 0) {
        s_base[0] = (tot_sc & 0xFFFFu) ? atomicAdd(&st->n_sel, tot_sc & 0xFFFFu) : 0u;
        s_base[1] = (tot_sc >> 16) ? atomicAdd(&st->n_cand, tot_sc >> 16) : 0u;
        s_base[2] = (p.full && tot_comp) ? atomicAdd(&st->n_comp, tot_comp) : 0u;
      }
      __syncthreads();
      uint32_t psel = s_base[0] + (inc_sc & 0xFFFFu) - nsel;
      uint32_t pcand = s_base[1] + (inc_sc >> 16) - ncand;
      uint32_t pcomp = s_base[2] + inc_comp - ncomp;
      __syncthreads();
#pragma unroll
      for (int u = 0; u < kPass2PerThread; ++u) {
        const int64_t t = tb + tid + u * kScanThreads;
        if (t >= t1) continue;
        const uint32_t d1 = key[u] >> 20;
        if (d1 > b1) {
          if (psel < (uint32_t)Nb) list[psel] = (int32_t)t;
          ++psel;
        } else if (d1 == b1) {
          if (pcand < (uint32_t)Nb) {
            ct[pcand] = (int32_t)t;
            ck[pcand] = key[u];
          }
          ++pcand;
          atomicAdd(&h2[(key[u] >> 8) & 0xFFFu], 1u);
        } else if (p.full) {
          if (pcomp < (uint32_t)Nb) list[Nb - 1 - (int64_t)pcomp] = (int32_t)t;
          ++pcomp;
          cmax = max(cmax, key[u]);
        }
      }
    }
    if (p.full) {
      cmax = warp_umax(cmax);
      if ((tid & 31) == 0 && cmax) atomicMax(&st->max_comp, cmax);
    }
    __syncthreads();
  });
}

// ------------------------------------------------------------- final_kernel
// One CTA per query head.
__global__ void __launch_bounds__(kScanThreads) final_kernel(DecodeParams p) {
  __shared__ uint32_t s_tmp[48];
  __shared__ uint32_t sh[2048];
  __shared__ uint32_t s_base[4];
  const int r = blockIdx.x, tid = threadIdx.x;
  const int b = r / p.Hq;
  const int Nb = p.lens[b];
  const uint32_t k = (uint32_t)p.kcnt[b];
  sdk_select_state* st = p.st + r;
  const uint32_t n_cand = st->n_cand;
  const uint32_t n_above = st->n_above;
  if (st->n_sel != n_above || n_above >= k || n_cand == 0u) {
    if (tid == 0) record_error(p.hdr, SDK_ERR_DEVICE_CHECK, 0x20000000u | r);
    return;
  }
  const uint32_t* ck = p.cand_key + (int64_t)r * p.L;
  const int32_t* ct = p.cand_t + (int64_t)r * p.L;
  int32_t* list = p.list + (int64_t)r * p.L;
  const uint32_t k1 = k - n_above;  // rank inside the pass-1 bucket

  // digit 2 (bits 19..8) from the global histogram
  uint32_t b2, above2, cnt2, b3, above3, cnt3;
  bool bad;
  block_find_desc<4096>(p.hist2 + (int64_t)r * 4096, k1, s_tmp, b2, above2, cnt2, bad);
  if (bad) {
    if (tid == 0) record_error(p.hdr, SDK_ERR_DEVICE_CHECK, 0x21000000u | r);
    return;
  }
  const uint32_t k2 = k1 - above2;
  // digit 3 (bits 7..0) over the candidates in bucket b2
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

  // With more ties than places, the places go to the lowest token indices:
  // radix-select the eq_take-th smallest token index among the ties
  // (digits 31..21, 20..10, 9..0; bins stored in reverse so the descending
  // search walks ascending token indices).
  uint32_t t_cut = 0xFFFFFFFFu;
  if (eq_total > eq_take) {
    uint32_t prefix = 0u, rank = eq_take;
    const int shifts[3] = {21, 10, 0};
    const int widths[3] = {11, 11, 10};
    for (int ps = 0; ps < 3; ++ps) {
      const int sh_lo = shifts[ps], wbits = widths[ps];
      const uint32_t nb = 1u << wbits;
      for (int i = tid; i < 2048; i += kScanThreads) sh[i] = 0u;
      __syncthreads();
      for (uint32_t i = tid; i < n_cand; i += kScanThreads) {
        if (ck[i] != T) continue;
        const uint32_t t = (uint32_t)ct[i];
        const uint32_t hi = (ps == 0) ? 0u : (t >> (sh_lo + wbits));
        if (hi != prefix) continue;
        const uint32_t dg = (t >> sh_lo) & (nb - 1u);
        atomicAdd(&sh[2047u - dg], 1u);
      }
      __syncthreads();
      uint32_t bin, above, cnt;
      block_find_desc<2048>(sh, rank, s_tmp, bin, above, cnt, bad);
      if (bad) {
        if (tid == 0) record_error(p.hdr, SDK_ERR_DEVICE_CHECK, 0x23000000u | r);
        return;
      }
      const uint32_t dg = 2047u - bin;
      prefix = (prefix << wbits) | dg;
      rank -= above;
    }
    t_cut = prefix;  // the eq_take-th smallest tie index
  }

  // classify the candidates; write selected to the front, the rest (with
  // full_softmax) to the back of the list
  uint32_t cmax = 0u;
  for (uint32_t i0 = 0; i0 < n_cand; i0 += kScanThreads) {
    const uint32_t i = i0 + tid;
    uint32_t key = 0u, t = 0u;
    bool sel = false, comp = false;
    if (i < n_cand) {
      key = ck[i];
      t = (uint32_t)ct[i];
      sel = key > T || (key == T && t <= t_cut);
      comp = !sel;
    }
    uint32_t tot_s, tot_c;
    const uint32_t inc = block_incl_scan((sel ? 1u : 0u) | ((comp && p.full) ? 0x10000u : 0u),
                                         s_tmp, &tot_s);
    (void)tot_c;
    if (tid == 0) {
      s_base[0] = atomicAdd(&st->n_sel, tot_s & 0xFFFFu);
      s_base[1] = p.full ? atomicAdd(&st->n_comp, tot_s >> 16) : 0u;
    }
    __syncthreads();
    if (sel) {
      const uint32_t pos = s_base[0] + (inc & 0xFFFFu) - 1u;
      if (pos < k) list[pos] = (int32_t)t;
      else record_error(p.hdr, SDK_ERR_DEVICE_CHECK, 0x26000000u | r);
    }
    if (comp && p.full) {
      const uint32_t pos = s_base[1] + (inc >> 16) - 1u;
      if (pos < (uint32_t)Nb) list[Nb - 1 - (int64_t)pos] = (int32_t)t;
      else record_error(p.hdr, SDK_ERR_DEVICE_CHECK, 0x27000000u | r);
      cmax = max(cmax, key);
    }
    __syncthreads();
  }
  if (p.full) {
    cmax = warp_umax(cmax);
    if ((tid & 31) == 0 && cmax) atomicMax(&st->max_comp, cmax);
  }
  __syncthreads();
  if (tid == 0) {
    st->kth_key = T;
    st->eq_total = eq_total;
    st->eq_taken = eq_take;
    __threadfence();
    if (st->n_sel != k) record_error(p.hdr, SDK_ERR_DEVICE_CHECK, 0x24000000u | r);
    if (p.full && st->n_sel + st->n_comp != (uint32_t)Nb)
      record_error(p.hdr, SDK_ERR_DEVICE_CHECK, 0x25000000u | r);
  }
}

// ----------------------------------------------------------- rescore_kernel
__global__ void __launch_bounds__(kScanThreads, 1) rescore_kernel(DecodeParams p) {
  extern __shared__ float4 smem4[];
  float* sq = reinterpret_cast<float*>(smem4);
  const int n = p.n, tid = threadIdx.x;
  const int64_t total = p.sel_off[p.B];
  const int64_t G0 = total * blockIdx.x / gridDim.x;
  const int64_t G1 = total * (blockIdx.x + 1) / gridDim.x;

  for_segments(p.sel_off, p.kcnt, p.B, G0, G1,
               [&](int b, int h, int64_t i0, int64_t i1) {
    const int r = b * p.Hq + h, kvh = h / p.g;
    const float* qdr = p.qd + (int64_t)r * n;
    const bool stage = (i1 - i0) * p.khigh >= (int64_t)(n / 2);
    if (stage) stage_row(sq, qdr, n);
    __syncthreads();
    const float* src = stage ? sq : qdr;
    const uint4* rec = reinterpret_cast<const uint4*>(
        p.k_full + ((int64_t)b * p.Hkv + kvh) * p.cap * kAtoms);
    const int32_t* list = p.list + (int64_t)r * p.L;
    float* out = p.sel_score + (int64_t)r * p.L;
    float smax = -INFINITY;
    const int Nb = p.lens[b];
    for (int64_t i = i0 + tid; i < i1; i += kScanThreads) {
      const int64_t t = list[i];
      if (t < 0 || t >= Nb) {
        record_error(p.hdr, SDK_ERR_DEVICE_CHECK, 0x30000000u | r);
        out[i] = -INFINITY;
        continue;
      }
      uint4 wv[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) wv[c] = __ldcs(rec + t * 4 + c);
      const uint32_t* wd = reinterpret_cast<const uint32_t*>(wv);
      float s = 0.0f;
#pragma unroll
      for (int j = 0; j < kAtoms; ++j) {
        if (j >= p.khigh) break;
        const uint32_t idx = word_idx(wd[j]);
        if (idx >= (uint32_t)n) {
          record_error(p.hdr, SDK_ERR_DEVICE_CHECK, idx);
          continue;
        }
        s = fmaf(word_coef(wd[j]), src[idx], s);
      }
      s *= p.scale;
      out[i] = s;
      smax = fmaxf(smax, s);
    }
    smax = warp_max(smax);
    if ((tid & 31) == 0 && smax > -INFINITY)
      atomicMax(&p.st[r].max_score, score_key(smax));
    __syncthreads();
  });
}

// ------------------------------------------------------------- value_kernel
__global__ void __launch_bounds__(kScanThreads, 1) value_kernel(DecodeParams p) {
  extern __shared__ float4 smem4[];
  float* sw = reinterpret_cast<float*>(smem4);
  __shared__ float s_red[32];
  const int n = p.n, tid = threadIdx.x;
  const int64_t total = p.dom_off[p.B];
  const int64_t G0 = total * blockIdx.x / gridDim.x;
  const int64_t G1 = total * (blockIdx.x + 1) / gridDim.x;

  for_segments(p.dom_off, p.dcnt, p.B, G0, G1,
               [&](int b, int h, int64_t i0, int64_t i1) {
    const int r = b * p.Hq + h, kvh = h / p.g;
    const sdk_select_state* st = p.st + r;
    const int k = p.kcnt[b];
    float m = key_score(st->max_score);
    if (p.full && st->n_comp > 0u) m = fmaxf(m, p.scale * key_score(st->max_comp));
    const bool smem_w = (i1 - i0) * kAtoms >= (int64_t)(n / 2);
    if (smem_w) {
      for (int i = tid; i < n; i += kScanThreads) sw[i] = 0.0f;
      __syncthreads();
    }
    float* wdst = smem_w ? sw : p.w + (int64_t)r * n;
    const uint4* rec = reinterpret_cast<const uint4*>(
        p.v_full + ((int64_t)b * p.Hkv + kvh) * p.cap * kAtoms);
    const int32_t* list = p.list + (int64_t)r * p.L;
    const float* ss = p.sel_score + (int64_t)r * p.L;
    const uint32_t* keys = p.keys + (int64_t)r * p.L;
    float z = 0.0f;
    const int Nb = p.lens[b];
    for (int64_t i = i0 + tid; i < i1; i += kScanThreads) {
      const int64_t t = list[i];
      if (t < 0 || t >= Nb) {
        record_error(p.hdr, SDK_ERR_DEVICE_CHECK, 0x31000000u | r);
        continue;
      }
      const float logit = (i < k) ? ss[i] : p.scale * key_score(keys[t]);
      const float e = expf(logit - m);
      z += e;
      uint4 wv[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) wv[c] = __ldcs(rec + t * 4 + c);
      const uint32_t* wd = reinterpret_cast<const uint32_t*>(wv);
#pragma unroll
      for (int j = 0; j < kAtoms; ++j) {
        const uint32_t idx = word_idx(wd[j]);
        if (idx >= (uint32_t)n) {
          record_error(p.hdr, SDK_ERR_DEVICE_CHECK, idx);
          continue;
        }
        atomicAdd(&wdst[idx], e * word_coef(wd[j]));
      }
    }
    z = warp_sum(z);
    if ((tid & 31) == 0) s_red[tid >> 5] = z;
    __syncthreads();
    if (tid == 0) {
      float zz = 0.0f;
      for (int i = 0; i < kScanThreads / 32; ++i) zz += s_red[i];
      atomicAdd(&p.st[r].z, zz);
    }
    if (smem_w) {
      float* gw = p.w + (int64_t)r * n;
      for (int i = tid; i < n; i += kScanThreads) {
        const float v = sw[i];
        if (v != 0.0f) atomicAdd(&gw[i], v);
      }
    }
    __syncthreads();
  });
}

// --------------------------------------------------------------- out_kernel
// part[tile][r][k] = sum_{a in tile} w[r][a] D_V[a][k]   (128-atom tiles,
// 32-row blocks).
template <int D>
__global__ void __launch_bounds__(256) out_kernel(DecodeParams p) {
  extern __shared__ float4 smem4[];
  float* Ds = reinterpret_cast<float*>(smem4);  // [128][D]
  float* Ws = Ds + 128 * D;                     // [128][32]
  const int n = p.n, R = p.R, tid = threadIdx.x;
  const int a0 = blockIdx.x * 128, r0 = blockIdx.y * 32;
  for (int e = tid; e < 128 * (D / 8); e += 256) {
    const int a = e / (D / 8), c = e % (D / 8);
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (a0 + a < n)
      v = __ldg(reinterpret_cast<const uint4*>(p.dv + (int64_t)(a0 + a) * D) + c);
    float4* d = reinterpret_cast<float4*>(Ds + a * D + c * 8);
    d[0] = make_float4(bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y));
    d[1] = make_float4(bf16_lo(v.z), bf16_hi(v.z), bf16_lo(v.w), bf16_hi(v.w));
  }
  for (int e = tid; e < 128 * 32; e += 256) {
    const int r = e & 31, a = e >> 5;
    Ws[a * 32 + r] = (r0 + r < R && a0 + a < n) ? p.w[(int64_t)(r0 + r) * n + a0 + a] : 0.0f;
  }
  __syncthreads();
  constexpr int C = D / 32;
  const int tk = tid & 31, tr = tid >> 5;
  float acc[4][C];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int c = 0; c < C; ++c) acc[i][c] = 0.0f;
#pragma unroll 4
  for (int a = 0; a < 128; ++a) {
    float dv[C];
    if constexpr (C == 4) {
      const float4 v = *reinterpret_cast<const float4*>(Ds + a * D + tk * 4);
      dv[0] = v.x; dv[1] = v.y; dv[2] = v.z; dv[3] = v.w;
    } else {
      const float2 v = *reinterpret_cast<const float2*>(Ds + a * D + tk * 2);
      dv[0] = v.x; dv[1] = v.y;
    }
    const float4 wv = *reinterpret_cast<const float4*>(Ws + a * 32 + 4 * tr);
    const float wr[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int c = 0; c < C; ++c) acc[i][c] = fmaf(wr[i], dv[c], acc[i][c]);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = r0 + 4 * tr + i;
    if (r >= R) continue;
    float* dst = p.part + ((int64_t)blockIdx.x * R + r) * D + tk * C;
#pragma unroll
    for (int c = 0; c < C; ++c) dst[c] = acc[i][c];
  }
}

__global__ void out_reduce_kernel(DecodeParams p) {
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t total = (int64_t)p.R * p.d;
  if (e >= total) return;
  const int r = (int)(e / p.d);
  float s = 0.0f;
  for (int t = 0; t < p.n_out_tiles; ++t) s += p.part[((int64_t)t * p.R) * p.d + e];
  p.out[e] = s / p.st[r].z;
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
  const size_t tiles = (size_t)(n + 127) / 128;
  l.part = take(tiles * R * d * 4);
  l.total = off;
  return l;
}

static int grid_for(int64_t work, int64_t per_cta, int cap_ctas) {
  int64_t g = (work + per_cta - 1) / per_cta;
  if (g < 1) g = 1;
  if (g > cap_ctas) g = cap_ctas;
  return (int)g;
}

sdk_status launch_decode(const DecodeParams& p0, cudaStream_t stream) {
  DecodeParams p = p0;
  const int sms = num_sms();
  const size_t qd_smem = (size_t)((p.n + 3) & ~3) * 4;
  cudaError_t e;

  // qd + zeroing
  {
    dim3 grid((p.n + 63) / 64, (p.R + 31) / 32);
    if (p.d == 128) qd_kernel<128><<<grid, 256, 0, stream>>>(p);
    else qd_kernel<64><<<grid, 256, 0, stream>>>(p);
  }
  // klow scan
  {
    const size_t smem = qd_smem + 4096 * 4;
    static bool attr = false;
    if (!attr) {
      cudaFuncSetAttribute(klow_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
      cudaFuncSetAttribute(rescore_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
      cudaFuncSetAttribute(value_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
      cudaFuncSetAttribute(out_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
      cudaFuncSetAttribute(out_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
      attr = true;
    }
    const int g = grid_for(p.tok_off[p.B], 2048, sms);
    klow_kernel<<<g, kScanThreads, smem, stream>>>(p);
  }
  {
    const int g = grid_for(p.tok_off[p.B], 4096, 2 * sms);
    pass2_kernel<<<g, kScanThreads, 0, stream>>>(p);
  }
  final_kernel<<<p.R, kScanThreads, 0, stream>>>(p);
  {
    const int g = grid_for(p.sel_off[p.B], 1024, sms);
    rescore_kernel<<<g, kScanThreads, qd_smem, stream>>>(p);
  }
  {
    const int g = grid_for(p.dom_off[p.B], 1024, sms);
    value_kernel<<<g, kScanThreads, qd_smem, stream>>>(p);
  }
  {
    dim3 grid(p.n_out_tiles, (p.R + 31) / 32);
    const size_t smem = (size_t)128 * p.d * 4 + 128 * 32 * 4;
    if (p.d == 128) out_kernel<128><<<grid, 256, smem, stream>>>(p);
    else out_kernel<64><<<grid, 256, smem, stream>>>(p);
  }
  {
    const int64_t tot = (int64_t)p.R * p.d;
    out_reduce_kernel<<<(unsigned)((tot + 255) / 256), 256, 0, stream>>>(p);
  }
  e = cudaGetLastError();
  return e == cudaSuccess ? SDK_OK : SDK_ERR_CUDA;
}

}  // namespace sdk
