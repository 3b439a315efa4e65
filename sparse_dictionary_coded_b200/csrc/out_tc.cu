// out += w D_V on the 5th-generation tensor cores (decode step D6).
//
// out[r][c] = sum_a w[r][a] D_V[a][c], computed transposed: out^T = D_V^T
// w^T with M = head_dim (128; 64-dim heads use the lower half), N = up to
// 128 query rows, K = the n atoms (split over the CTAs).  Both operands come
// straight from global memory with TMA, in the layouts they already have:
//   * A = a chunk of 64 atoms of D_V (bf16 [atom][head_dim], head_dim
//     contiguous), read as an MN-major operand: two 64-element halves of the
//     head dimension, each 64 atom rows of 128 bytes (128-byte swizzle);
//   * B = the same 64 atoms of the three bf16 parts of w (attend writes w as
//     w_0 + w_1 + w_2, the remainder below 2^-24 |w| for normal values),
//     K-major ([part][row][atom], one 3-D box per chunk).
// One thread streams the chunks through a ring of kStages stages, one thread
// issues 3 x 4 tcgen05.mma (M=128, N, K=16) per chunk into one fp32 TMEM
// accumulator, and the four warps read it back (thread = output column).
// CTAs run in clusters of kWCluster consecutive atom ranges: after the
// MMAs each CTA parks its partial tile [N][head_dim] in shared memory, and
// CTA k of the cluster sums a quarter of the rows over the cluster's tiles
// (distributed shared memory) and adds it into `out` (zeroed by the QD
// kernel of the call) with vector reductions.  Every mbarrier wait is
// bounded (1 s): on expiry the CTA records SDK_ERR_TIMEOUT, contributes a
// zero tile and still completes the cluster's synchronisation.
#include <cooperative_groups.h>

#include "tc_ptx.cuh"

namespace sdk {
namespace tc {

constexpr int kWM = 128;        // MMA M (head_dim rows of out^T)
constexpr int kWChunk = 64;     // atoms per stage: one 128-byte row of a w part
constexpr int kWThreads = 128;  // producer lane, MMA lane, four epilogue warps
constexpr int kWSplit = 3;      // bf16 parts of w
constexpr int kWCluster = 4;    // CTAs whose partial tiles are summed on chip

template <int N>
struct WCfg {
  static constexpr int kABytes = kWM * kWChunk * 2;          // two 8 KB halves
  static constexpr int kBBytes = kWSplit * N * kWChunk * 2;  // [part][N][64]
  static constexpr int kStage = kABytes + kBBytes;
  static constexpr int kStages = N <= 64 ? 4 : 3;
  static constexpr int kPStride = kWM + 4;                   // partial tile row (floats)
  static_assert(N * kPStride * 4 <= kStages * kStage, "partial tile must fit the ring");
  static constexpr int kOffBar = kStages * kStage;
  static constexpr int kNumBars = 2 * kStages + 1;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmem = kOffMisc + 16 + 1024;         // + 1024-byte alignment slack
  static_assert(kSmem <= 232448, "exceeds the 227 KB shared memory of one sm_100 CTA");
  static constexpr uint32_t kTmemCols = N < 32 ? 32u : (uint32_t)N;
  // instruction descriptor: D f32, A and B bf16, A MN-major (bit 15),
  // B K-major, N, M = 128
  static constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) |
                                     ((uint32_t)(N >> 3) << 17) | ((uint32_t)(kWM >> 4) << 24);
};

template <int D, int N>
__global__ void __launch_bounds__(kWThreads, 1)
    out_tc_kernel(const __grid_constant__ CUtensorMap vmap, const __grid_constant__ CUtensorMap wmap,
                  DecodeParams p) {
  using C = WCfg<N>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_smem_1k(smem_raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile uint32_t* s_abort = misc + 0;
  volatile uint32_t* s_tmem = misc + 1;
  auto bar_full = [&](int s) { return smem_u32(&bars[s]); };
  auto bar_empty = [&](int s) { return smem_u32(&bars[C::kStages + s]); };
  const uint32_t bar_done = smem_u32(&bars[2 * C::kStages]);
  const uint32_t s0 = smem_u32(smem);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int R = p.R;
  const int nchunks = (p.n + kWChunk - 1) / kWChunk;
  const int c0 = (int)((int64_t)nchunks * blockIdx.x / gridDim.x);
  const int c1 = (int)((int64_t)nchunks * (blockIdx.x + 1) / gridDim.x);
  const int r0 = blockIdx.y * N;

  if (tid == 0) {
    *s_abort = 0u;
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(bar_full(s), 1);
      mbar_init(bar_empty(s), 1);
    }
    mbar_init(bar_done, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32((const void*)s_tmem)),
                 "r"(C::kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (D < kWM) {
    // 64-dim heads: the upper half of every A stage (rows 64..127 of out^T)
    // stays zero; TMA writes only the lower half
    for (int s = 0; s < C::kStages; ++s)
      for (int e = tid; e < 8192 / 16; e += kWThreads)
        reinterpret_cast<uint4*>(smem + s * C::kStage + 8192)[e] = make_uint4(0u, 0u, 0u, 0u);
    fence_proxy_async();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, issued_mask = 0, last_phase = 0;
      bool ok = true;
      for (int c = c0; c < c1; ++c) {
        if (!mbar_wait(bar_empty(stage), phase ^ 1u, s_abort)) {
          ok = false;
          break;
        }
        const uint32_t st = s0 + stage * C::kStage;
        mbar_expect_tx(bar_full(stage), (uint32_t)(D * kWChunk * 2 + C::kBBytes));
        tma_load_2d(st, &vmap, 0, c * kWChunk, bar_full(stage));
        if (D > 64) tma_load_2d(st + 8192, &vmap, 64, c * kWChunk, bar_full(stage));
        tma_load_3d(st + C::kABytes, &wmap, c * kWChunk, r0, 0, bar_full(stage));
        issued_mask |= 1u << stage;
        last_phase = (last_phase & ~(1u << stage)) | (phase << stage);
        if (++stage == C::kStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) {
        record_error(p.hdr, SDK_ERR_TIMEOUT, 0x54000000u | blockIdx.x);
        *s_abort = 1u;
      }
      // every copy issued has landed before the CTA may leave
      for (int s = 0; s < C::kStages; ++s)
        if (issued_mask & (1u << s)) {
          uint32_t dummy = 0u;
          mbar_wait(bar_full(s), (last_phase >> s) & 1u, &dummy, 100000000ull);
        }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true, issued = false;
      for (int c = c0; c < c1; ++c) {
        if (!mbar_wait(bar_full(stage), phase, s_abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t sa = s0 + stage * C::kStage, sb = sa + C::kABytes;
#pragma unroll
        for (int s = 0; s < kWSplit; ++s)
#pragma unroll
          for (int ks = 0; ks < kWChunk / 16; ++ks) {
            // A: 16 atoms = two 8-row swizzle atoms (2048 bytes); the two
            // halves of the head dimension are 8192 bytes apart.  B: 16
            // atoms = 32 bytes along the K-major rows of part s.
            tc_mma(tmem, smem_desc_mn(sa + ks * 2048, 8192u, 1024u),
                   smem_desc(sb + s * (N * 128) + ks * 32), C::kIdesc,
                   (issued || s > 0 || ks > 0) ? 1u : 0u);
          }
        issued = true;
        tc_commit(bar_empty(stage));
        if (++stage == C::kStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) {
        record_error(p.hdr, SDK_ERR_TIMEOUT, 0x55000000u | blockIdx.x);
        *s_abort = 1u;
      }
      // arrives once every MMA issued has completed (at once if none was)
      tc_commit(bar_done);
    }
  }
  __syncwarp();

  // ------------------------------------------------------------ epilogue
  // thread i = TMEM lane i = column i of out (row i of out^T)
  uint32_t never = 0u;
  const bool got = lane == 0 ? mbar_wait(bar_done, 0u, &never) : true;
  const bool done = __shfl_sync(0xffffffffu, got ? 1 : 0, 0) != 0;
  if (!done && lane == 0) record_error(p.hdr, SDK_ERR_TIMEOUT, 0x56000000u | blockIdx.x);
  tc_fence_after();
  __syncthreads();   // the ring is free: the partial tile [N][kPStride] reuses it
  const bool have = done && c1 > c0 && *s_abort == 0u;
  float* part = reinterpret_cast<float*>(smem);
  {
    const int i = warp * 32 + lane;
#pragma unroll
    for (int cb = 0; cb < N; cb += 32) {
      uint32_t v[32];
      if (have && warp * 32 < D) {
        tmem_ld32(tmem + ((uint32_t)(warp * 32) << 16) + cb, v);
        tmem_ld_wait();
      } else {
#pragma unroll
        for (int u = 0; u < 32; ++u) v[u] = 0u;
      }
      if (i < D) {
#pragma unroll
        for (int u = 0; u < 32; ++u)
          if (cb + u < N) part[(cb + u) * C::kPStride + i] = __uint_as_float(v[u]);
      }
    }
  }
  tc_fence_before();
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  cluster.sync();
  {
    const int cr = (int)cluster.block_rank();
    constexpr int kRowsPer = N / kWCluster;
    const float* parts[kWCluster];
#pragma unroll
    for (int k = 0; k < kWCluster; ++k) parts[k] = cluster.map_shared_rank(part, k);
    for (int e = tid; e < kRowsPer * (D / 4); e += kWThreads) {
      const int i = cr * kRowsPer + e / (D / 4), c4 = e % (D / 4);
      if (r0 + i >= R) continue;
      float4 x[kWCluster];
#pragma unroll
      for (int k = 0; k < kWCluster; ++k)
        x[k] = *reinterpret_cast<const float4*>(parts[k] + i * C::kPStride + 4 * c4);
      float4 acc = x[0];
#pragma unroll
      for (int k = 1; k < kWCluster; ++k) {
        acc.x += x[k].x;
        acc.y += x[k].y;
        acc.z += x[k].z;
        acc.w += x[k].w;
      }
      float* dst = p.out + (int64_t)(r0 + i) * D + 4 * c4;
      asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(dst), "f"(acc.x),
                   "f"(acc.y), "f"(acc.z), "f"(acc.w)
                   : "memory");
    }
  }
  cluster.sync();   // the peers' tiles are read before any CTA leaves
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(C::kTmemCols)
                 : "memory");
  }
}

// Launches out_tc_kernel<D, N> over ty row tiles and up to gx atom ranges
// (fewer when fewer clusters of this kernel fit the device at once).
template <int D, int N>
static cudaError_t launch_w(const CUtensorMap& vmap, const CUtensorMap& wmap, const DecodeParams& p,
                            int gx, int ty, cudaStream_t stream) {
  static unsigned long long attr_set = 0ull;
  static int max_clusters[64];
  int dev = 0;
  cudaGetDevice(&dev);
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kWThreads);
  cfg.dynamicSmemBytes = WCfg<N>::kSmem;
  cfg.stream = stream;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = kWCluster;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  if (device_needs_setup(&attr_set)) {
    cudaFuncSetAttribute(out_tc_kernel<D, N>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         WCfg<N>::kSmem);
    int mc = 0;
    cfg.gridDim = dim3(kWCluster);
    if (cudaOccupancyMaxActiveClusters(&mc, out_tc_kernel<D, N>, &cfg) != cudaSuccess) {
      cudaGetLastError();
      mc = 0;
    }
    if (dev >= 0 && dev < 64) max_clusters[dev] = mc;
    device_setup_done(&attr_set);
  }
  const int mc = (dev >= 0 && dev < 64) ? max_clusters[dev] : 0;
  if (mc > 0 && gx * ty > mc * kWCluster) gx = mc * kWCluster / ty / kWCluster * kWCluster;
  if (gx < kWCluster) gx = kWCluster;
  cfg.gridDim = dim3((unsigned)gx, (unsigned)ty);
  cfg.blockDim = dim3(kWThreads);
  return cudaLaunchKernelEx(&cfg, out_tc_kernel<D, N>, vmap, wmap, p);
}

}  // namespace tc

// w D_V on the tensor cores; *taken = false when the path is not available
// (head_dim other than 64/128, rows of w that are not a multiple of 16
// bytes, or no driver entry point for tensor maps).
sdk_status launch_out_tc(const DecodeParams& p, cudaStream_t stream, bool* taken) {
  *taken = false;
  if ((p.d != 64 && p.d != 128) || (p.n % 8) != 0 || p.R < 1) return SDK_OK;
  auto fn = tc::encode_fn();
  if (fn == nullptr) return SDK_OK;
  // D_V [n][d] bf16: boxes of 64 head-dim elements x 64 atoms
  CUtensorMap vmap, wmap;
  {
    const cuuint64_t dims[2] = {(cuuint64_t)p.d, (cuuint64_t)p.n};
    const cuuint64_t strides[1] = {(cuuint64_t)p.d * 2};
    const cuuint32_t box[2] = {64u, (cuuint32_t)tc::kWChunk};
    const cuuint32_t estr[2] = {1u, 1u};
    if (fn(&vmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(p.dv), dims, strides,
           box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return SDK_OK;
  }
  // rows per tile: the smallest of 32 / 64 / 128 that holds R (128 above)
  const int N = p.R <= 32 ? 32 : (p.R <= 64 ? 64 : 128);
  {
    // w parts [3][R][n] bf16: boxes of 64 atoms x N rows x 3 parts (rows
    // past R read as zero)
    const cuuint64_t dims[3] = {(cuuint64_t)p.n, (cuuint64_t)p.R, (cuuint64_t)tc::kWSplit};
    const cuuint64_t strides[2] = {(cuuint64_t)p.n * 2, (cuuint64_t)p.R * p.n * 2};
    const cuuint32_t box[3] = {(cuuint32_t)tc::kWChunk, (cuuint32_t)N, (cuuint32_t)tc::kWSplit};
    const cuuint32_t estr[3] = {1u, 1u, 1u};
    if (fn(&wmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, p.w, dims, strides, box, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return SDK_OK;
  }
  *taken = true;
  // atom ranges: whole clusters, about one CTA per SM over all row tiles
  const int ty = (p.R + N - 1) / N;
  const int nchunks = (p.n + tc::kWChunk - 1) / tc::kWChunk;
  int gx = num_sms() / ty;
  if (gx > nchunks) gx = nchunks;
  gx = gx / tc::kWCluster * tc::kWCluster;
  cudaError_t e;
  if (p.d == 128)
    e = N == 32 ? tc::launch_w<128, 32>(vmap, wmap, p, gx, ty, stream)
        : N == 64 ? tc::launch_w<128, 64>(vmap, wmap, p, gx, ty, stream)
                  : tc::launch_w<128, 128>(vmap, wmap, p, gx, ty, stream);
  else
    e = N == 32 ? tc::launch_w<64, 32>(vmap, wmap, p, gx, ty, stream)
        : N == 64 ? tc::launch_w<64, 64>(vmap, wmap, p, gx, ty, stream)
                  : tc::launch_w<64, 128>(vmap, wmap, p, gx, ty, stream);
  return e == cudaSuccess ? SDK_OK : SDK_ERR_CUDA;
}

}  // namespace sdk
