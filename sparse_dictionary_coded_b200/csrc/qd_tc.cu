// QD = q D_K^T on the 5th-generation tensor cores (decode step D1).
//
// QD[r][a] = sum_k q[r][k] D_K[a][k] for R query rows against all n atoms,
// computed transposed: QD^T = D_K q^T with M = 128 atoms per tile, N = up
// to 128 query rows, K = head_dim.  The A operand is the bf16 dictionary
// tile itself (TMA, 128-byte swizzle, K-major); q is fp32, and to keep fp32
// accuracy each element is split into three bf16 parts, q = q_hi + q_mid +
// q_lo (each the bf16 rounding of what the previous parts leave; the
// remainder is below 2^-24 |q| for normal values), written by the CTA's
// threads as three K-major B operands.  The three products with the exact
// bf16 atoms accumulate in fp32 in tensor memory: 3 x (head_dim / 16) MMAs
// per atom tile.
//
// One CTA per (row tile of N query rows, strided set of 128-atom tiles), 6
// warps: warp 0 streams dictionary tiles with TMA through a kQStages ring
// from the first instruction on, warps 1..5 meanwhile zero the per-call
// state and build the q parts, then warp 1 issues tcgen05.mma (M=128, N,
// K=16) into one of two TMEM accumulators and warps 2..5 read an
// accumulator back (tcgen05.ld, thread = atom, columns = query rows) and
// store it to QD, 128 consecutive atoms of a row per warp store.  Rows past
// R are zero in the B operand and are not stored.  Every mbarrier wait is
// bounded (1 s); on expiry the CTA records SDK_ERR_TIMEOUT and stops.
//
// Like the CUDA-core QD kernel this first kernel of a decode call also
// zeroes the per-head selection state, both histograms and `out`.
#include "tc_ptx.cuh"

namespace sdk {
namespace tc {

constexpr int kQAtoms = 128;    // MMA M
constexpr int kQStages = 3;
constexpr int kQThreads = 192;  // producer, MMA issuer, 4 epilogue warps
constexpr int kQSplit = 3;      // bf16 parts of q

template <int D, int N>
struct QCfg {
  static constexpr int KB = D / 64;                     // 128-byte K blocks
  static constexpr int KSTEPS = D / 16;
  static constexpr int kStageBytes = kQAtoms * D * 2;   // one dictionary tile
  static constexpr int kBBytes = N * D * 2;             // one bf16 part of q
  static constexpr int kOffB = kQStages * kStageBytes;
  static constexpr int kOffBar = kOffB + kQSplit * kBBytes;
  static constexpr int kNumBars = 2 * kQStages + 2 + 2 + 1;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmem = kOffMisc + 64 + 1024;   // + 1024-byte alignment slack
  static_assert(kSmem <= 232448, "exceeds the 227 KB shared memory of one sm_100 CTA");
  static constexpr uint32_t kTmemCols = 2 * N < 32 ? 32u : (uint32_t)(2 * N);
  // instruction descriptor: D f32, A and B bf16, both K-major, N, M = 128
  static constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) |
                                     ((uint32_t)(N >> 3) << 17) | ((uint32_t)(kQAtoms >> 4) << 24);
};

template <int D, int N>
__global__ void __launch_bounds__(kQThreads, 1)
    qd_tc_kernel(const __grid_constant__ CUtensorMap tmap, DecodeParams p) {
  using C = QCfg<D, N>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_smem_1k(smem_raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile uint32_t* s_abort = misc + 0;
  volatile uint32_t* s_tmem = misc + 1;
  const uint32_t sA = smem_u32(smem);
  const uint32_t sB = smem_u32(smem + C::kOffB);
  auto bar_full = [&](int s) { return smem_u32(&bars[s]); };
  auto bar_empty = [&](int s) { return smem_u32(&bars[kQStages + s]); };
  auto bar_tfull = [&](int b) { return smem_u32(&bars[2 * kQStages + b]); };
  auto bar_tempty = [&](int b) { return smem_u32(&bars[2 * kQStages + 2 + b]); };
  const uint32_t bar_done = smem_u32(&bars[2 * kQStages + 4]);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n = p.n, R = p.R;
  const int r0 = blockIdx.y * N;
  const int n_atom_tiles = (n + kQAtoms - 1) / kQAtoms;

  if (tid == 0) {
    *s_abort = 0u;
    for (int s = 0; s < kQStages; ++s) {
      mbar_init(bar_full(s), 1);
      mbar_init(bar_empty(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar_tfull(b), 1);
      mbar_init(bar_tempty(b), 4);
    }
    mbar_init(bar_done, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32((const void*)s_tmem)),
                 "r"(C::kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
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
      for (int a = blockIdx.x; ok && a < n_atom_tiles; a += gridDim.x) {
        if (!mbar_wait(bar_empty(stage), phase ^ 1u, s_abort)) {
          ok = false;
          break;
        }
        mbar_expect_tx(bar_full(stage), (uint32_t)C::kStageBytes);
#pragma unroll
        for (int kb = 0; kb < C::KB; ++kb)
          tma_load_2d(sA + stage * C::kStageBytes + kb * (kQAtoms * 128), &tmap, kb * 64,
                      a * kQAtoms, bar_full(stage));
        issued_mask |= 1u << stage;
        last_phase = (last_phase & ~(1u << stage)) | (phase << stage);
        if (++stage == kQStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) {
        record_error(p.hdr, SDK_ERR_TIMEOUT, 0x50000000u | blockIdx.x);
        *s_abort = 1u;
      }
      for (int s = 0; s < kQStages; ++s)
        if (issued_mask & (1u << s)) {
          uint32_t dummy = 0u;
          mbar_wait(bar_full(s), (last_phase >> s) & 1u, &dummy, 100000000ull);
        }
    }
    return;
  }

  // ---- warps 1..5, while the first tiles load: the per-call state
  // (selection state, histograms, out) and the B operands
  {
    constexpr int kT = kQThreads - 32;
    const int t = tid - 32;
    const int64_t nthr = (int64_t)gridDim.x * gridDim.y * kT;
    const int64_t g0 = ((int64_t)blockIdx.y * gridDim.x + blockIdx.x) * kT + t;
    // both histograms, 16-byte stores (the radix selection path only)
    const int64_t hquads = p.bracket ? 0 : (int64_t)R * 1024;
    for (int64_t e = g0; e < hquads; e += nthr) {
      reinterpret_cast<uint4*>(p.hist1)[e] = make_uint4(0u, 0u, 0u, 0u);
      reinterpret_cast<uint4*>(p.hist2)[e] = make_uint4(0u, 0u, 0u, 0u);
    }
    for (int64_t e = g0; e < (int64_t)R * D; e += nthr) p.out[e] = 0.0f;
    for (int64_t e = g0; e < (int64_t)R; e += nthr) {
      sdk_select_state st = {};
      st.k = (uint32_t)p.kcnt[e / p.Hq];
      p.st[e] = st;
    }
    // B operands: the three bf16 parts of the tile's query rows in the
    // 128-byte-swizzled K-major layout (8 elements = one 16-byte chunk;
    // chunk c of K block kb of row i lives at kb*N*128 + i*128 +
    // ((c^(i&7))*16)); rows past R are zero
    // (the loads of kQBatch chunks are in flight before the first is used)
    constexpr int kItems = N * (D / 8), kQBatch = 8;
    for (int e0 = t; e0 < kItems; e0 += kQBatch * kT) {
      float4 x[kQBatch][2];
#pragma unroll
      for (int u = 0; u < kQBatch; ++u) {
        const int e = e0 + u * kT;
        const int i = e / (D / 8), kc = e % (D / 8);
        if (e < kItems && r0 + i < R) {   // q is 16-byte aligned (checked by the API)
          const float4* src =
              reinterpret_cast<const float4*>(p.q + (int64_t)(r0 + i) * D + kc * 8);
          x[u][0] = __ldg(src);
          x[u][1] = __ldg(src + 1);
        } else {
          x[u][0] = x[u][1] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
#pragma unroll
      for (int u = 0; u < kQBatch; ++u) {
        const int e = e0 + u * kT;
        if (e >= kItems) break;
        const int i = e / (D / 8), kc = e % (D / 8);
        const float v[8] = {x[u][0].x, x[u][0].y, x[u][0].z, x[u][0].w,
                            x[u][1].x, x[u][1].y, x[u][1].z, x[u][1].w};
        uint32_t w[kQSplit][4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float a0 = v[2 * c], a1 = v[2 * c + 1];
#pragma unroll
          for (int s = 0; s < kQSplit; ++s) {
            const __nv_bfloat162 h = __floats2bfloat162_rn(a0, a1);
            w[s][c] = *reinterpret_cast<const uint32_t*>(&h);
            a0 -= __low2float(h);       // exact: the rounding error of a0
            a1 -= __high2float(h);
          }
        }
        const int kb = kc >> 3, c16 = kc & 7;
#pragma unroll
        for (int s = 0; s < kQSplit; ++s) {
          uint4* dst = reinterpret_cast<uint4*>(smem + C::kOffB + s * C::kBBytes +
                                                kb * (N * 128) + i * 128 + ((c16 ^ (i & 7)) << 4));
          *dst = make_uint4(w[s][0], w[s][1], w[s][2], w[s][3]);
        }
      }
    }
    fence_proxy_async();   // generic-proxy stores of B before the MMAs read them
    asm volatile("bar.sync 1, %0;" ::"r"(kT) : "memory");
  }

  if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    if (lane == 0) {
      tc_fence_after();
      int stage = 0;
      uint32_t phase = 0, tbuf = 0, tphase = 0;
      bool ok = true, issued = false;
      for (int a = blockIdx.x; ok && a < n_atom_tiles; a += gridDim.x) {
        if (!mbar_wait(bar_full(stage), phase, s_abort) ||
            !mbar_wait(bar_tempty(tbuf), tphase ^ 1u, s_abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t abase = sA + stage * C::kStageBytes;
        const uint32_t d_tmem = tmem + tbuf * N;
#pragma unroll
        for (int s = 0; s < kQSplit; ++s)
#pragma unroll
          for (int ks = 0; ks < C::KSTEPS; ++ks) {
            const uint32_t aoff = (ks >> 2) * (kQAtoms * 128) + (ks & 3) * 32;
            const uint32_t boff = (ks >> 2) * (N * 128) + (ks & 3) * 32;
            tc_mma(d_tmem, smem_desc(abase + aoff), smem_desc(sB + s * C::kBBytes + boff),
                   C::kIdesc, (s > 0 || ks > 0) ? 1u : 0u);
          }
        issued = true;
        tc_commit(bar_empty(stage));
        tc_commit(bar_tfull(tbuf));
        if (++stage == kQStages) {
          stage = 0;
          phase ^= 1u;
        }
        tbuf ^= 1u;
        if (tbuf == 0u) tphase ^= 1u;
      }
      if (!ok) {
        record_error(p.hdr, SDK_ERR_TIMEOUT, 0x51000000u | blockIdx.x);
        *s_abort = 1u;
      }
      if (issued) {
        tc_commit(bar_done);
        uint32_t dummy = 0u;
        mbar_wait(bar_done, 0u, &dummy, 100000000ull);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    // warp w reads TMEM lanes 32*(w%4) .. +31: one atom per thread, the
    // tile's query rows along the columns
    const int quarter = warp & 3;
    uint32_t tbuf = 0, tphase = 0;
    for (int a = blockIdx.x; a < n_atom_tiles; a += gridDim.x) {
      // lane 0 waits (false on timeout or abort), the warp follows its answer
      const bool got = lane == 0 ? mbar_wait(bar_tfull(tbuf), tphase, s_abort) : true;
      if (!__shfl_sync(0xffffffffu, got ? 1 : 0, 0)) {
        if (lane == 0 && !*s_abort) {
          record_error(p.hdr, SDK_ERR_TIMEOUT, 0x52000000u | blockIdx.x);
          *s_abort = 1u;
        }
        break;
      }
      tc_fence_after();
      const int atom = a * kQAtoms + quarter * 32 + lane;
      const uint32_t taddr = tmem + ((uint32_t)(quarter * 32) << 16) + tbuf * N;
#pragma unroll
      for (int cb = 0; cb < N; cb += 32) {
        uint32_t v[32];
        tmem_ld32(taddr + cb, v);
        tmem_ld_wait();
        if (cb + 32 >= N) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar_tempty(tbuf));
        }
        if (atom < n) {
          float* dst = p.qd + (int64_t)(r0 + cb) * n + atom;
#pragma unroll
          for (int c = 0; c < 32; ++c)
            if (r0 + cb + c < R) dst[(int64_t)c * n] = __uint_as_float(v[c]);
        }
      }
      tbuf ^= 1u;
      if (tbuf == 0u) tphase ^= 1u;
    }
  }

  asm volatile("bar.sync 1, %0;" ::"r"(kQThreads - 32) : "memory");
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(C::kTmemCols)
                 : "memory");
  }
}

template <int D, int N>
static void qd_launch(const CUtensorMap& map, const DecodeParams& p, dim3 grid,
                      cudaStream_t stream) {
  static unsigned long long attr_set = 0ull;
  if (device_needs_setup(&attr_set)) {
    cudaFuncSetAttribute(qd_tc_kernel<D, N>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         QCfg<D, N>::kSmem);
    device_setup_done(&attr_set);
  }
  qd_tc_kernel<D, N><<<grid, kQThreads, QCfg<D, N>::kSmem, stream>>>(map, p);
}

}  // namespace tc

// QD on the tensor cores; *taken = false when the path is not available
// (head_dim other than 64/128, or no driver entry point for tensor maps).
sdk_status launch_qd_tc(const DecodeParams& p, cudaStream_t stream, bool* taken) {
  *taken = false;
  if (p.d != 64 && p.d != 128) return SDK_OK;
  auto fn = tc::encode_fn();
  if (fn == nullptr) return SDK_OK;
  CUtensorMap map;
  const cuuint64_t dims[2] = {(cuuint64_t)p.d, (cuuint64_t)p.n};
  const cuuint64_t strides[1] = {(cuuint64_t)p.d * 2};
  const cuuint32_t box[2] = {64u, (cuuint32_t)tc::kQAtoms};
  const cuuint32_t estr[2] = {1u, 1u};
  CUresult cr = fn(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(p.dk), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (cr != CUDA_SUCCESS) return SDK_OK;   // fall back to the CUDA-core kernel
  *taken = true;
  // rows per tile: the smallest of 32 / 64 / 128 that holds R (128 above)
  const int N = p.R <= 32 ? 32 : (p.R <= 64 ? 64 : 128);
  const int ty = (p.R + N - 1) / N;
  const int tiles = (p.n + tc::kQAtoms - 1) / tc::kQAtoms;
  int gx = num_sms() / ty;
  if (gx < 1) gx = 1;
  if (gx > tiles) gx = tiles;
  const dim3 grid((unsigned)gx, (unsigned)ty);
  if (p.d == 128) {
    if (N == 32) tc::qd_launch<128, 32>(map, p, grid, stream);
    else if (N == 64) tc::qd_launch<128, 64>(map, p, grid, stream);
    else tc::qd_launch<128, 128>(map, p, grid, stream);
  } else {
    if (N == 32) tc::qd_launch<64, 32>(map, p, grid, stream);
    else if (N == 64) tc::qd_launch<64, 64>(map, p, grid, stream);
    else tc::qd_launch<64, 128>(map, p, grid, stream);
  }
  return cudaGetLastError() == cudaSuccess ? SDK_OK : SDK_ERR_CUDA;
}

}  // namespace sdk
