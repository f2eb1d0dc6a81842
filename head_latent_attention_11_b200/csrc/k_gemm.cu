// k_gemm.cu — a2 (wq_b with the RoPE epilogue), a4 (W_UK absorption) and a8 (W_UV expansion):
// D[m, n] = sum_k A[g][m, k] · B[g][n, k] on the 5th-generation tensor cores.
//
// "DeepSeek-V3.2-Exp · Query heads": q = c^Q · wq_b, split per head into 128 content and 64
// rotary features, rotary half rotated (formula block, Explanation, mla-queries excerpt).
// "DeepSeek-V3.2-Exp · Attention update", mla-decode excerpt: q_nope absorbed through
// wkv_b[:, :nope] ("bshd,hdc->bshc") and the attention result expanded through wkv_b[:, -v:]
// ("bshc,hdc->bshd").
//
// All three are "weights as M" GEMMs: A is a weight matrix (128 weight rows per tile, K-major),
// B holds the token rows (K-major), so decode batches of a few tokens still fill the 128-row MMA.
// The kernel is persistent: one CTA per SM walks the output tiles ("units": batch g = head for
// a4/a8, 128-row weight tile, BN-token tile) round-robin, and its TMA ring streams K slabs
// continuously across unit boundaries, so weight streaming never drains between tiles.
//   warp 0      TMA producer: 64-wide K slabs of A (128 x 64) and B (BN x 64), 128-byte swizzle,
//               into a STAGES-deep shared-memory ring (~200 KB, one CTA per SM);
//   warp 1      allocates TMEM and issues tcgen05.mma (M=128, N=BN, K=16) per slab into one of
//               two accumulators (units alternate), committing each slab back to the producer
//               and each finished unit to the epilogue;
//   warps 2-5   epilogue: tcgen05.ld the fp32 accumulator (thread = weight row), apply RoPE for
//               the rotary rows of wq_b (partner of a pair = neighbouring lane), store bf16,
//               hand the accumulator back — overlapping the next unit's MMAs.
#include "internal.h"
#include "tc100.cuh"

namespace mla {

namespace {

constexpr int kGemmThreads = 192;
constexpr int kSlabA = 128 * 64 * 2;   // 16 KB

template <int BN>
struct GemmTile {
  static constexpr int kSlabB = BN * 64 * 2;
  static constexpr int kTmemCols = 2 * BN < 32 ? 32 : 2 * BN;   // two accumulators
};

template <int BN, int STAGES>
constexpr int gemm_smem_bytes() {
  return 1024 /*align slack*/ + STAGES * (kSlabA + GemmTile<BN>::kSlabB) + 256 /*barriers*/;
}

__device__ __forceinline__ void epi_store(const GemmParams& p, int g, int m, int n, float v,
                                          float partner) {
  if (p.epi == kEpiWqbRope) {
    const int h = m / kDq, j = m - h * kDq;
    if (j < kDn) {
      p.out0[static_cast<size_t>(n) * p.ld_n0 + static_cast<size_t>(h) * kDn + j] =
          __float2bfloat16_rn(v);
    } else {
      const int jj = j - kDn;                 // 0..63, pair jj/2
      const float2 cs = p.rope_tab[static_cast<size_t>(n) * kRopePairs + (jj >> 1)];
      // q is a bf16 tensor before the rotation (bf16 wq_b output, "Query heads" mla-queries)
      v = bf16_round(v);
      partner = bf16_round(partner);
      float r;
      if ((jj & 1) == 0) r = v * cs.x - partner * cs.y;      // x0 cos - x1 sin
      else r = partner * cs.y + v * cs.x;                     // x0 sin + x1 cos
      p.out1[(static_cast<size_t>(n) * kHPad + h) * kDk + kC + jj] = __float2bfloat16_rn(r);
    }
  } else {
    p.out0[static_cast<size_t>(n) * p.ld_n0 + static_cast<size_t>(g) * p.ld_g0 + m] =
        __float2bfloat16_rn(v);
  }
}

struct Unit {
  int g, m0, n0;
};

__device__ __forceinline__ Unit unit_of(int u, int mt, int nt, int BN) {
  // tokens fastest: consecutive units share a weight tile (its re-reads hit L2)
  Unit r;
  const int n = u % nt;
  const int rest = u / nt;
  r.m0 = (rest % mt) * 128;
  r.g = rest / mt;
  r.n0 = n * BN;
  return r;
}

// Work split: CTA c takes units c, c + G, c + 2G, ... (G = grid size).
struct Sched {
  int units, G, u;
  __device__ void init(int nunits, int grid, int cta) {
    units = nunits;
    G = grid;
    u = cta;
  }
  __device__ bool next(int& unit) {
    if (u >= units) return false;
    unit = u;
    u += G;
    return true;
  }
};

template <int BN, int STAGES>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_bf16_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const GemmParams p, const int batches) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * kSlabA;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sB + STAGES * GemmTile<BN>::kSlabB);
  uint64_t* full = bars;
  uint64_t* empty = bars + STAGES;
  uint64_t* acc_full = bars + 2 * STAGES;        // [2]
  uint64_t* acc_empty = bars + 2 * STAGES + 2;   // [2]
  uint64_t* drain = bars + 2 * STAGES + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  pdl_launch_dependents();
  const int warp = warp_id();
  const int nk = p.K / 64;
  const int mt = p.M / 128;
  const int nt = (p.N + BN - 1) / BN;
  const int total = batches * mt * nt;
  Guard guard{abort_flag, p.status};
  Sched sched;
  sched.init(total, gridDim.x, blockIdx.x);

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 128);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) tmem_alloc(tmem_slot, GemmTile<BN>::kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (elect_one()) {
      const uint64_t pol_w = policy_evict_first();   // weights are read once per call
      // The weight slabs of the first ring pass do not depend on the previous kernel: issue them
      // before waiting for it, so weight streaming overlaps that kernel's tail.
      int npre = 0;
      {
        Sched pre = sched;
        int u;
        while (npre < STAGES && pre.next(u)) {
          const Unit un = unit_of(u, mt, nt, BN);
          for (int j = 0; j < nk && npre < STAGES; ++j, ++npre) {
            mbar_arrive_expect_tx(&full[npre], kSlabA + GemmTile<BN>::kSlabB);
            tma_load_3d_hint(sA + npre * kSlabA, &tmA, &full[npre], j * 64, un.m0 + p.a_row_off,
                             un.g, pol_w);
          }
        }
      }
      pdl_wait();
      int ks = 0;
      bool ok = true;
      int u;
      while (ok && sched.next(u)) {
        const Unit un = unit_of(u, mt, nt, BN);
        for (int j = 0; j < nk; ++j, ++ks) {
          const int s = ks % STAGES;
          if (ks >= npre) {
            if (ks >= STAGES && !mbar_wait(&empty[s], ((ks / STAGES) - 1) & 1, guard)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(&full[s], kSlabA + GemmTile<BN>::kSlabB);
            tma_load_3d_hint(sA + s * kSlabA, &tmA, &full[s], j * 64, un.m0 + p.a_row_off, un.g,
                             pol_w);
          }
          tma_load_3d(sB + s * GemmTile<BN>::kSlabB, &tmB, &full[s], j * 64, un.g, un.n0);
        }
      }
      if (guard.aborted()) {
        // drain the loads still in flight before the CTA's shared memory goes away
        int dummy = 0;
        Guard dr{reinterpret_cast<volatile int*>(&dummy), p.status};
        for (int k = ks > STAGES ? ks - STAGES : 0; k < ks; ++k)
          mbar_wait(&full[k % STAGES], (k / STAGES) & 1, dr);
      }
    }
  } else if (warp == 1) {
    if (elect_one()) {
      const uint32_t idesc = idesc_bf16(128, BN, false, false);
      int ks = 0, si = 0;
      bool ok = true;
      int u;
      while (ok && sched.next(u)) {
        const int ab = si & 1;
        if (si >= 2 && !mbar_wait(&acc_empty[ab], ((si >> 1) - 1) & 1, guard)) break;
        tc_fence_after();
        const uint32_t d = tmem + ab * BN;
        for (int j = 0; j < nk; ++j, ++ks) {
          const int s = ks % STAGES;
          if (!mbar_wait(&full[s], (ks / STAGES) & 1, guard)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + s * kSlabA);
          const uint32_t b0 = smem_u32(sB + s * GemmTile<BN>::kSlabB);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            umma_bf16(d, smem_desc_sw128(a0 + kk * 32, 16, 1024),
                      smem_desc_sw128(b0 + kk * 32, 16, 1024), idesc, (j | kk) != 0);
          }
          umma_commit(&empty[s]);
        }
        if (!ok) break;
        umma_commit(&acc_full[ab]);
        ++si;
      }
      umma_commit(drain);
    }
  } else {
    // epilogue warps 2..5 → TMEM lane quadrant warp % 4
    pdl_wait();   // outputs may be read by the kernel before this one
    const int quad = warp & 3;
    const int row = quad * 32 + static_cast<int>(lane_id());
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    int si = 0;
    int u;
    while (sched.next(u)) {
      const Unit un = unit_of(u, mt, nt, BN);
      const int ab = si & 1;
      if (!warp_wait(&acc_full[ab], (si >> 1) & 1, guard)) break;
      tc_fence_after();
      const int m = un.m0 + row;
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 16) {
        if (un.n0 + c0 >= p.N) break;   // uniform across the warp
        float v[16];
        tmem_ld16(tmem + lane_off + ab * BN + c0, v);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float partner = __shfl_xor_sync(0xffffffffu, v[i], 1);
          const int n = un.n0 + c0 + i;
          if (n < p.N) epi_store(p, un.g, m, n, v[i], partner);
        }
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[ab]);
      ++si;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    int dummy = 0;
    Guard dr{reinterpret_cast<volatile int*>(&dummy), p.status};
    mbar_wait(drain, 0, dr);   // no MMA still writes the accumulators
    tc_fence_after();
    tmem_dealloc(tmem, GemmTile<BN>::kTmemCols);
  }
}

int g_num_sms = 0;

template <int BN, int STAGES>
cudaError_t launch_gemm_t(const CUtensorMap& ta, const CUtensorMap& tb, const GemmParams& p,
                          int batches, cudaStream_t s, bool pdl) {
  if (g_num_sms == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&g_num_sms, cudaDevAttrMultiProcessorCount, dev);
    if (g_num_sms <= 0) g_num_sms = 1;
  }
  const int total = batches * (p.M / 128) * ((p.N + BN - 1) / BN);
  const int grid = total < g_num_sms ? total : g_num_sms;
  LaunchCfg lc(dim3(grid), dim3(kGemmThreads), gemm_smem_bytes<BN, STAGES>(), s, pdl);
  return cudaLaunchKernelEx(&lc.cfg, gemm_bf16_kernel<BN, STAGES>, ta, tb, p, batches);
}

template <int BN, int STAGES>
cudaError_t set_attr() {
  static_assert(gemm_smem_bytes<BN, STAGES>() <= 232448, "shared memory budget");
  return cudaFuncSetAttribute(gemm_bf16_kernel<BN, STAGES>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize,
                              gemm_smem_bytes<BN, STAGES>());
}

}  // namespace

// Tile choice: BN covers the token count up to 256; the ring fills ~200 KB of shared memory.
cudaError_t launch_gemm(const CUtensorMap& ta, const CUtensorMap& tb, const GemmParams& p,
                        int batches, cudaStream_t s, bool pdl) {
  if (p.N <= 32) return launch_gemm_t<32, 10>(ta, tb, p, batches, s, pdl);
  if (p.N <= 64) return launch_gemm_t<64, 8>(ta, tb, p, batches, s, pdl);
  if (p.N <= 128) return launch_gemm_t<128, 6>(ta, tb, p, batches, s, pdl);
  return launch_gemm_t<256, 4>(ta, tb, p, batches, s, pdl);
}

cudaError_t gemm_prepare() {
  cudaError_t e;
  if ((e = set_attr<32, 10>()) != cudaSuccess) return e;
  if ((e = set_attr<64, 8>()) != cudaSuccess) return e;
  if ((e = set_attr<128, 6>()) != cudaSuccess) return e;
  return set_attr<256, 4>();
}

// W_UK^T copy made once at set-up: w_ukt[h][c][d] = wkv_b[h*256 + d][c], d < 128, so that the
// absorption GEMM reads its weight K-major like the other two.
__global__ void transpose_uk_kernel(const bf16* __restrict__ wkv_b, bf16* __restrict__ w_ukt) {
  __shared__ bf16 tile[32][33];
  const int h = blockIdx.z;
  const int c0 = blockIdx.x * 32, d0 = blockIdx.y * 32;
  const int tx = threadIdx.x, ty = threadIdx.y;   // 32 x 8
  for (int i = ty; i < 32; i += 8)
    tile[i][tx] = wkv_b[(static_cast<size_t>(h) * (kDn + kDv) + d0 + i) * kC + c0 + tx];
  __syncthreads();
  for (int i = ty; i < 32; i += 8)
    w_ukt[(static_cast<size_t>(h) * kC + c0 + i) * kDn + d0 + tx] = tile[tx][i];
}

cudaError_t launch_transpose_uk(const bf16* wkv_b, bf16* w_ukt, int n_heads, cudaStream_t s) {
  dim3 grid(kC / 32, kDn / 32, n_heads), block(32, 8);
  transpose_uk_kernel<<<grid, block, 0, s>>>(wkv_b, w_ukt);
  return cudaGetLastError();
}

}  // namespace mla
