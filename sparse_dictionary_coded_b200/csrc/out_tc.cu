// out += w D_V on the 5th-generation tensor cores (decode step D6).
//
// out[r][c] = sum_a w[r][a] D_V[a][c]: M = R query rows, N = head_dim,
// K = n atoms.  Each CTA takes 128 atoms (split-K) and up to 128 rows:
//   * the atoms' value rows (bf16 [128 atoms][head_dim], 32 KB) and the rows'
//     weights (fp32 [rows][128 atoms]) arrive with cp.async;
//   * the value tile is transposed in shared memory into the K-major,
//     128-byte-swizzled B operand ([head_dim][128 atoms]); the weights are
//     split per element into three bf16 parts (w = w_hi + w_mid + w_lo, the
//     remainder below 2^-24 |w| for normal values) forming three A operands;
//   * one thread issues 3 x 8 tcgen05.mma (M=128, N=head_dim, K=16) into one
//     TMEM accumulator (fp32);
//   * four warps read it back (one row per thread) into shared memory;
//   * CTAs run in clusters of kOCluster adjacent atom slices: CTA k of a
//     cluster sums rows [k 128/kOCluster, (k+1) 128/kOCluster) over the
//     cluster's partial tiles (distributed shared memory) and adds them into
//     `out` (zeroed by the QD kernel of the call) with vector reductions, so
//     every output element takes n / (128 kOCluster) global reductions.
// The single wait on the MMA completion is bounded (1 s; SDK_ERR_TIMEOUT).
#include <cooperative_groups.h>

#include "tc_ptx.cuh"

namespace sdk {
namespace tc {

constexpr int kORows = 128;    // MMA M
constexpr int kOAtoms = 128;   // K per CTA
constexpr int kOThreads = 128;
constexpr int kOSplit = 3;
constexpr int kOCluster = 4;   // CTAs (atom slices) summed on chip per reduction

template <int D>
struct OCfg {
  static constexpr int kBBytes = D * kOAtoms * 2;         // B operand, bf16 [D][atoms]
  static constexpr int kABytes = kORows * kOAtoms * 2;    // one bf16 part [rows][atoms]
  static constexpr int kVBytes = kOAtoms * D * 2;         // staged values [atoms][D]
  static constexpr int kWBytes = kORows * kOAtoms * 4;    // staged weights fp32
  static constexpr int kOffB = 0;
  static constexpr int kOffA = kOffB + kBBytes;
  static constexpr int kOffV = kOffA + kOSplit * kABytes;
  static constexpr int kOffW = kOffV + kVBytes;
  // the partial tile fp32 [128][D + 4] reuses the value and weight staging
  static constexpr int kPStride = D + 4;
  static_assert(kORows * kPStride * 4 <= kVBytes + kWBytes, "partial tile must fit");
  static constexpr int kOffBar = kOffW + kWBytes;
  static constexpr int kOffMisc = kOffBar + 8;
  static constexpr int kSmem = kOffMisc + 16 + 1024;     // + 1024-byte alignment slack
  static_assert(kSmem <= 232448, "exceeds the 227 KB shared memory of one sm_100 CTA");
};

// Instruction descriptor: D f32, A and B bf16, both K-major, N = D, M = 128.
template <int D>
struct OIdesc {
  static constexpr uint32_t value = (1u << 4) | (1u << 7) | (1u << 10) |
                                    ((uint32_t)(D >> 3) << 17) | ((uint32_t)(kORows >> 4) << 24);
};

// byte offset of the 16-byte chunk (row, chunk c) in a K-major
// 128-byte-swizzled operand with 128 rows per 64-element K block
__device__ __forceinline__ uint32_t swz_off(int row, int c, int rows) {
  return (uint32_t)((c >> 3) * (rows * 128) + row * 128 + (((c & 7) ^ (row & 7)) << 4));
}

template <int D>
__global__ void __launch_bounds__(kOThreads, 1) out_tc_kernel(DecodeParams p) {
  using C = OCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_smem_1k(smem_raw);
  const uint32_t bar = smem_u32(smem + C::kOffBar);
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile uint32_t* s_tmem = misc;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n = p.n, R = p.R;
  const int a0 = blockIdx.x * kOAtoms;
  const int r0 = blockIdx.y * kORows;

  if (tid == 0) {
    mbar_init(bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32((const void*)s_tmem)),
                 "r"(D)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  // stage the value rows and the weights (all copies of a thread in flight)
  const uint16_t* dv = p.dv + (int64_t)a0 * D;
  uint4* vst = reinterpret_cast<uint4*>(smem + C::kOffV);
  for (int e = tid; e < kOAtoms * (D / 8); e += kOThreads) {
    const int a = e / (D / 8);
    const bool v = a0 + a < n;
    cp_async16(vst + e, reinterpret_cast<const uint4*>(v ? dv : p.dv) + (v ? e : 0), v);
  }
  float* wst = reinterpret_cast<float*>(smem + C::kOffW);
  for (int e = tid; e < kORows * (kOAtoms / 4); e += kOThreads) {
    const int i = e / (kOAtoms / 4), c4 = e % (kOAtoms / 4);
    const bool v = r0 + i < R && a0 + 4 * c4 + 3 < n;
    const float* src = v ? p.w + (int64_t)(r0 + i) * n + a0 + 4 * c4 : p.w;
    cp_async16(wst + i * kOAtoms + 4 * c4, src, v);
  }
  cp_async_commit();
  cp_async_wait<0>();
  __syncthreads();
  // weights of a partial last tile that do not fill 16 bytes: plain loads
  if (a0 + kOAtoms > n) {
    for (int e = tid; e < kORows * kOAtoms; e += kOThreads) {
      const int i = e / kOAtoms, a = e % kOAtoms;
      const int c4 = a >> 2;
      const bool vec = r0 + i < R && a0 + 4 * c4 + 3 < n;
      if (!vec) wst[e] = (r0 + i < R && a0 + a < n) ? p.w[(int64_t)(r0 + i) * n + a0 + a] : 0.0f;
    }
    __syncthreads();
  }
  // B operand: transpose [atoms][D] -> K-major [D][atoms]; thread takes
  // 8 consecutive atoms of one column c (one 16-byte chunk of the operand)
  const uint16_t* vs = reinterpret_cast<const uint16_t*>(smem + C::kOffV);
  for (int e = tid; e < D * (kOAtoms / 8); e += kOThreads) {
    const int c = e % D, ch = e / D;            // c: column (operand row), ch: atom chunk
    uint32_t w4[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const uint32_t lo = vs[(ch * 8 + 2 * u) * D + c];
      const uint32_t hi = vs[(ch * 8 + 2 * u + 1) * D + c];
      w4[u] = lo | (hi << 16);
    }
    *reinterpret_cast<uint4*>(smem + C::kOffB + swz_off(c, ch, D)) =
        make_uint4(w4[0], w4[1], w4[2], w4[3]);
  }
  // A operands: three bf16 parts of the weights
  for (int e = tid; e < kORows * (kOAtoms / 8); e += kOThreads) {
    const int i = e / (kOAtoms / 8), ch = e % (kOAtoms / 8);
    const float4 x0 = *reinterpret_cast<const float4*>(wst + i * kOAtoms + ch * 8);
    const float4 x1 = *reinterpret_cast<const float4*>(wst + i * kOAtoms + ch * 8 + 4);
    const float v[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
    uint32_t w[kOSplit][4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      float a0f = v[2 * u], a1f = v[2 * u + 1];
#pragma unroll
      for (int s = 0; s < kOSplit; ++s) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(a0f, a1f);
        w[s][u] = *reinterpret_cast<const uint32_t*>(&h);
        a0f -= __low2float(h);
        a1f -= __high2float(h);
      }
    }
#pragma unroll
    for (int s = 0; s < kOSplit; ++s)
      *reinterpret_cast<uint4*>(smem + C::kOffA + s * C::kABytes + swz_off(i, ch, kORows)) =
          make_uint4(w[s][0], w[s][1], w[s][2], w[s][3]);
  }
  fence_proxy_async();   // generic stores of the operands before the MMAs read them
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;
  if (tid == 0) {
    const uint32_t sA = smem_u32(smem + C::kOffA), sB = smem_u32(smem + C::kOffB);
#pragma unroll
    for (int s = 0; s < kOSplit; ++s)
#pragma unroll
      for (int ks = 0; ks < kOAtoms / 16; ++ks) {
        const uint32_t koffA = (ks >> 2) * (kORows * 128) + (ks & 3) * 32;
        const uint32_t koffB = (ks >> 2) * (D * 128) + (ks & 3) * 32;
        tc_mma(tmem, smem_desc(sA + s * C::kABytes + koffA), smem_desc(sB + koffB),
               OIdesc<D>::value, (s > 0 || ks > 0) ? 1u : 0u);
      }
    tc_commit(bar);
  }
  __syncwarp();
  // every warp waits for the accumulator (lane 0 waits, bounded)
  uint32_t never = 0u;
  const bool got = lane == 0 ? mbar_wait(bar, 0u, &never) : true;
  const bool ok = __shfl_sync(0xffffffffu, got ? 1 : 0, 0) != 0;
  if (!ok && lane == 0) record_error(p.hdr, SDK_ERR_TIMEOUT, 0x53000000u | blockIdx.x);
  tc_fence_after();
  // the accumulator into shared memory, one row per thread (zeros if the
  // MMAs timed out: the error is recorded, the cluster still completes)
  float* part = reinterpret_cast<float*>(smem + C::kOffV);
  {
    const int i = warp * 32 + lane;
#pragma unroll
    for (int c0 = 0; c0 < D; c0 += 32) {
      uint32_t v[32];
      if (ok) {
        tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + c0, v);
        tmem_ld_wait();
      } else {
#pragma unroll
        for (int u = 0; u < 32; ++u) v[u] = 0u;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u)
        *reinterpret_cast<uint4*>(part + i * C::kPStride + c0 + 4 * u) =
            make_uint4(v[4 * u], v[4 * u + 1], v[4 * u + 2], v[4 * u + 3]);
    }
  }
  tc_fence_before();
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  cluster.sync();
  // this CTA's rows of the cluster's sum, into `out`
  {
    const int cr = (int)cluster.block_rank();
    constexpr int kRowsPer = kORows / kOCluster;
    const float* parts[kOCluster];
#pragma unroll
    for (int k = 0; k < kOCluster; ++k) parts[k] = cluster.map_shared_rank(part, k);
    for (int e = tid; e < kRowsPer * (D / 4); e += kOThreads) {
      const int i = cr * kRowsPer + e / (D / 4), c4 = e % (D / 4);
      if (r0 + i >= R) continue;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int k = 0; k < kOCluster; ++k) {
        const float4 x = *reinterpret_cast<const float4*>(parts[k] + i * C::kPStride + 4 * c4);
        acc.x += x.x;
        acc.y += x.y;
        acc.z += x.z;
        acc.w += x.w;
      }
      float* dst = p.out + (int64_t)(r0 + i) * D + 4 * c4;
      asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(dst), "f"(acc.x),
                   "f"(acc.y), "f"(acc.z), "f"(acc.w)
                   : "memory");
    }
  }
  cluster.sync();   // the peers' tiles are read before any CTA leaves
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(D)
                 : "memory");
  }
}

}  // namespace tc

// w D_V on the tensor cores; *taken = false when not available.
sdk_status launch_out_tc(const DecodeParams& p, cudaStream_t stream, bool* taken) {
  *taken = false;
  // 16-byte weight copies need rows of a multiple of 4 atoms
  if ((p.d != 64 && p.d != 128) || (p.n & 3) != 0) return SDK_OK;
  *taken = true;
  static unsigned long long attr_set = 0ull;
  if (device_needs_setup(&attr_set)) {
    cudaFuncSetAttribute(tc::out_tc_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         tc::OCfg<128>::kSmem);
    cudaFuncSetAttribute(tc::out_tc_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         tc::OCfg<64>::kSmem);
    device_setup_done(&attr_set);
  }
  // atom slices rounded up to whole clusters (slices past n are zero)
  int slices = (p.n + tc::kOAtoms - 1) / tc::kOAtoms;
  slices = (slices + tc::kOCluster - 1) / tc::kOCluster * tc::kOCluster;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)slices, (unsigned)((p.R + tc::kORows - 1) / tc::kORows));
  cfg.blockDim = dim3(tc::kOThreads);
  cfg.dynamicSmemBytes = p.d == 128 ? tc::OCfg<128>::kSmem : tc::OCfg<64>::kSmem;
  cfg.stream = stream;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = tc::kOCluster;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  const cudaError_t e = p.d == 128 ? cudaLaunchKernelEx(&cfg, tc::out_tc_kernel<128>, p)
                                   : cudaLaunchKernelEx(&cfg, tc::out_tc_kernel<64>, p);
  return e == cudaSuccess ? SDK_OK : SDK_ERR_CUDA;
}

}  // namespace sdk
