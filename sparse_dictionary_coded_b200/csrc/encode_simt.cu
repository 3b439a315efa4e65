// Greedy pursuit encoder on CUDA cores, exact in fp32 ("LLM Inference in a
// Flash!", evolve.pub review, Summary: a projection-based greedy pursuit
// replaces OMP; the coefficient is the projection, no least-squares refit).
//
// One CTA encodes 64 vectors; the fp32 residuals stay in shared memory for
// all k_atoms steps.  Each step streams the dictionary through shared memory
// in 64-atom tiles; thread (tv, ta) computes the 4x4 correlations of
// vectors 4tv..4tv+3 with atoms 4ta..4ta+3 of the tile as fp32 FMA chains
// over k = 0..D-1, keeps the running best |c| (ties: lowest index), and a
// 16-lane shuffle reduction picks the winner per vector.  The correlation of
// the winner is its coefficient; r -= coef * d in fp32.
#include "sdk_internal.cuh"

namespace sdk {


constexpr int kSimtVecs = 64;

template <int D>
__global__ void __launch_bounds__(256) encode_simt_kernel(EncodeParams p) {
  extern __shared__ float4 smem4[];
  float* rT = reinterpret_cast<float*>(smem4);   // [D][64] residuals
  float* Dt = rT + D * kSimtVecs;                // [D][64] atom tile
  __shared__ int s_idx[kSimtVecs];
  __shared__ float s_coef[kSimtVecs];
  const int tid = threadIdx.x;
  const int64_t v0 = (int64_t)blockIdx.x * kSimtVecs;
  const int n = p.n;

  for (int e = tid; e < D * kSimtVecs; e += 256) {
    const int v = e & 63, k = e >> 6;
    float xv = 0.0f;
    if (v0 + v < p.n_vec) {
      const int64_t o = (v0 + v) * D + k;
      xv = p.x_dtype == SDK_F32 ? reinterpret_cast<const float*>(p.x)[o]
                                : bf16_lo(reinterpret_cast<const uint16_t*>(p.x)[o]);
    }
    rT[k * kSimtVecs + v] = xv;
  }

  const int ta = tid & 15, tv = tid >> 4;
  for (int j = 0; j < p.k_atoms; ++j) {
    float bestA[4], bestC[4];
    int bestI[4];
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      bestA[v] = -1.0f;
      bestC[v] = 0.0f;
      bestI[v] = 0;
    }
    for (int a0 = 0; a0 < n; a0 += 64) {
      __syncthreads();
      for (int e = tid; e < 64 * (D / 8); e += 256) {
        const int a = e & 63, c = e >> 6;
        uint4 w = make_uint4(0u, 0u, 0u, 0u);
        if (a0 + a < n)
          w = __ldg(reinterpret_cast<const uint4*>(p.dict + (int64_t)(a0 + a) * D) + c);
        float* col = Dt + (c * 8) * kSimtVecs + a;
        col[0 * kSimtVecs] = bf16_lo(w.x);
        col[1 * kSimtVecs] = bf16_hi(w.x);
        col[2 * kSimtVecs] = bf16_lo(w.y);
        col[3 * kSimtVecs] = bf16_hi(w.y);
        col[4 * kSimtVecs] = bf16_lo(w.z);
        col[5 * kSimtVecs] = bf16_hi(w.z);
        col[6 * kSimtVecs] = bf16_lo(w.w);
        col[7 * kSimtVecs] = bf16_hi(w.w);
      }
      __syncthreads();
      float acc[4][4];
#pragma unroll
      for (int v = 0; v < 4; ++v)
#pragma unroll
        for (int u = 0; u < 4; ++u) acc[v][u] = 0.0f;
#pragma unroll 4
      for (int k = 0; k < D; ++k) {
        const float4 dv = *reinterpret_cast<const float4*>(Dt + k * kSimtVecs + 4 * ta);
        const float4 rv = *reinterpret_cast<const float4*>(rT + k * kSimtVecs + 4 * tv);
        const float dd[4] = {dv.x, dv.y, dv.z, dv.w};
        const float rr[4] = {rv.x, rv.y, rv.z, rv.w};
#pragma unroll
        for (int v = 0; v < 4; ++v)
#pragma unroll
          for (int u = 0; u < 4; ++u) acc[v][u] = fmaf(rr[v], dd[u], acc[v][u]);
      }
#pragma unroll
      for (int v = 0; v < 4; ++v)
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int atom = a0 + 4 * ta + u;
          const float m = fabsf(acc[v][u]);
          if (atom < n && m > bestA[v]) {
            bestA[v] = m;
            bestC[v] = acc[v][u];
            bestI[v] = atom;
          }
        }
    }
    // reduce over the 16 lanes that share tv (ties: lower atom index)
#pragma unroll
    for (int v = 0; v < 4; ++v) {
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) {
        const float oa = __shfl_xor_sync(0xffffffffu, bestA[v], o);
        const float oc = __shfl_xor_sync(0xffffffffu, bestC[v], o);
        const int oi = __shfl_xor_sync(0xffffffffu, bestI[v], o);
        if (oa > bestA[v] || (oa == bestA[v] && oi < bestI[v])) {
          bestA[v] = oa;
          bestC[v] = oc;
          bestI[v] = oi;
        }
      }
      if (ta == 0) {
        s_idx[4 * tv + v] = bestI[v];
        s_coef[4 * tv + v] = bestC[v];
      }
    }
    __syncthreads();
    // residual update r -= coef * d_i* (fp32, one rounding per component)
    for (int e = tid; e < D * kSimtVecs; e += 256) {
      const int v = e & 63, k = e >> 6;
      const float d = bf16_lo(__ldg(p.dict + (int64_t)s_idx[v] * D + k));
      rT[k * kSimtVecs + v] = fmaf(-s_coef[v], d, rT[k * kSimtVecs + v]);
    }
    if (tid < kSimtVecs && v0 + tid < p.n_vec)
      p.codes[(v0 + tid) * p.k_atoms + j] = make_word(s_coef[tid], (uint32_t)s_idx[tid]);
  }
  __syncthreads();
  if (p.rsq != nullptr && tid < kSimtVecs && v0 + tid < p.n_vec) {
    float s = 0.0f;
    for (int k = 0; k < D; ++k) {
      const float r = rT[k * kSimtVecs + tid];
      s = fmaf(r, r, s);
    }
    p.rsq[v0 + tid] = s;
  }
}

sdk_status launch_encode_simt(const EncodeParams& p, int head_dim, cudaStream_t stream) {
  if (p.n_vec == 0) return SDK_OK;
  const unsigned grid = (unsigned)((p.n_vec + kSimtVecs - 1) / kSimtVecs);
  const size_t smem = (size_t)2 * head_dim * kSimtVecs * 4;
  static unsigned long long attr_set = 0ull;
  if (device_needs_setup(&attr_set)) {
    cudaFuncSetAttribute(encode_simt_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)(2 * 128 * kSimtVecs * 4));
    cudaFuncSetAttribute(encode_simt_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)(2 * 64 * kSimtVecs * 4));
    device_setup_done(&attr_set);
  }
  if (head_dim == 128) encode_simt_kernel<128><<<grid, 256, smem, stream>>>(p);
  else encode_simt_kernel<64><<<grid, 256, smem, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? SDK_OK : SDK_ERR_CUDA;
}

}  // namespace sdk
