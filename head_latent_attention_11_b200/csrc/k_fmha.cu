// k_fmha.cu — the prefill chunk in its non-absorbed form: multi-head attention with per-head keys
// and values rebuilt from the latent cache.
//
// "Kimi-K2 · value_states", mla-prefill excerpt: for every head the query is [q_nope ‖ q_pe], the
// key is [k_nope ‖ k_pe] with k_pe the shared rotary key of the cache and k_nope = W_UK kv, the
// value is W_UV kv; scores are scaled, the additive causal mask is applied, the softmax is taken
// in fp32 and mixes the values.
//
// The keys and values are rebuilt once per chunk by the GEMM kernel (kvb[key][h][0:128) = k_nope,
// [128:256) = v); this kernel computes, for one (sequence, head, 128-token query tile):
//   S = Q K^T (M = 128 tokens, N = 128 keys, K = 192: k_nope from kvb, k_pe from the cache),
//   causal mask (key j visible to token t iff j <= start_pos + t), online fp32 softmax,
//   O += P V (N = 128 value features), on the 5th-generation tensor cores with the accumulators
//   in TMEM: O [0,128) | two 128-column score/probability buffers [128,384).
// Warp roles: warp 0 TMA producer, warp 1 TMEM owner + MMA issuer (scores and P·V), warps 2-5
// softmax and epilogue (thread = query row = TMEM lane).  Key tiles stream through a two-stage
// ring (K 48 KB + V 32 KB per stage); the score MMA of tile j+1 runs while tile j is in the
// softmax.  Every wait is bounded.
#include "internal.h"
#include "tc100.cuh"

namespace mla {

namespace {

constexpr int kFN = 128;                    // keys per tile
constexpr int kFStages = 2;
constexpr int kFSlab = 128 * 64 * 2;        // 16 KB: 128 rows x 64 bf16 columns
constexpr int kFStageBytes = 5 * kFSlab;    // K: 3 slabs (k_nope 0-63, 64-127, k_pe), V: 2 slabs
constexpr int kFOffQ = 0;                   // Q: 3 slabs (q_nope 0-63, 64-127, q_pe)
constexpr int kFOffKV = kFOffQ + 3 * kFSlab;
constexpr int kFOffBar = kFOffKV + kFStages * kFStageBytes;
constexpr int kFmhaSmem = kFOffBar + 256 + 1024;
constexpr int kFThreads = 64 + 128;
constexpr uint32_t kFTmemO = 0, kFTmemS = 128;
constexpr float kFRescale = 8.0f;

struct FBars {
  uint64_t q_full;
  uint64_t kv_full[kFStages], kv_empty[kFStages];
  uint64_t s_full[2], p_full[2], pv_done[2];
  uint64_t drain;
  uint32_t tmem_slot;
  int abort_flag;
};
static_assert(sizeof(FBars) <= 256, "barrier block");
static_assert(kFmhaSmem <= 232448, "shared memory budget");

__global__ void __launch_bounds__(kFThreads, 1)
    fmha_prefill_kernel(const __grid_constant__ CUtensorMap tmQn,   // q_nope {128, H, rows}
                        const __grid_constant__ CUtensorMap tmQp,   // absorbed query {576, 128, rows}
                        const __grid_constant__ CUtensorMap tmKvb,  // kvb {H*256, keys, B}
                        const __grid_constant__ CUtensorMap tmPe,   // rotary cache {64, L, B}
                        const FmhaParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem + kFOffQ;
  uint8_t* sKV = smem + kFOffKV;
  FBars* bar = reinterpret_cast<FBars*>(smem + kFOffBar);

  pdl_launch_dependents();
  const int qt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int t0 = qt * 128;
  const int row0 = b * p.T + t0;                          // first query row of the tile
  const int last_pos = p.start_pos + min(t0 + 127, p.T - 1);
  const int ntiles = last_pos / kFN + 1;                  // key tiles any row of the tile sees
  const int warp = static_cast<int>(warp_id());
  Guard guard{reinterpret_cast<volatile int*>(&bar->abort_flag), p.status,
              p.wait_limit_ns ? p.wait_limit_ns : kWaitLimitNs};

  if (threadIdx.x == 0) {
    mbar_init(&bar->q_full, 1);
    for (int i = 0; i < kFStages; ++i) {
      mbar_init(&bar->kv_full[i], 1);
      mbar_init(&bar->kv_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar->s_full[i], 1);
      mbar_init(&bar->p_full[i], 128);
      mbar_init(&bar->pv_done[i], 1);
    }
    mbar_init(&bar->drain, 1);
    bar->abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmQn);
    tma_prefetch_desc(&tmQp);
    tma_prefetch_desc(&tmKvb);
    tma_prefetch_desc(&tmPe);
  }
  if (warp == 1) tmem_alloc(&bar->tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar->tmem_slot;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (elect_one()) {
      pdl_wait();   // queries and rebuilt keys / values come from the previous kernels
      mbar_arrive_expect_tx(&bar->q_full, 3 * kFSlab);
      tma_load_3d(sQ, &tmQn, &bar->q_full, 0, h, row0);
      tma_load_3d(sQ + kFSlab, &tmQn, &bar->q_full, 64, h, row0);
      tma_load_3d(sQ + 2 * kFSlab, &tmQp, &bar->q_full, kC, h, row0);
      int issued = 0;
      for (int j = 0; j < ntiles; ++j) {
        const int s = j % kFStages;
        if (j >= kFStages && !mbar_wait(&bar->kv_empty[s], ((j / kFStages) - 1) & 1, guard)) break;
        uint8_t* st = sKV + s * kFStageBytes;
        uint64_t* fb = &bar->kv_full[s];
        mbar_arrive_expect_tx(fb, kFStageBytes);
        const int key = j * kFN;
        tma_load_3d(st, &tmKvb, fb, h * 256, key, b);                 // k_nope 0-63
        tma_load_3d(st + kFSlab, &tmKvb, fb, h * 256 + 64, key, b);   // k_nope 64-127
        tma_load_3d(st + 2 * kFSlab, &tmPe, fb, 0, key, b);           // k_pe
        tma_load_3d(st + 3 * kFSlab, &tmKvb, fb, h * 256 + 128, key, b);   // v 0-63
        tma_load_3d(st + 4 * kFSlab, &tmKvb, fb, h * 256 + 192, key, b);   // v 64-127
        issued = j + 1;
      }
      if (guard.aborted()) {
        int dummy = 0;
        Guard drain{reinterpret_cast<volatile int*>(&dummy), p.status};
        mbar_wait(&bar->q_full, 0, drain);
        for (int j = issued > kFStages ? issued - kFStages : 0; j < issued; ++j)
          mbar_wait(&bar->kv_full[j % kFStages], (j / kFStages) & 1, drain);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    // Score MMA of tile j+1 is issued before P·V of tile j (it only needs the other score buffer),
    // so the softmax of tile j overlaps the tensor core's work on tile j+1.
    if (elect_one()) {
      const uint32_t idesc_qk = idesc_bf16(128, kFN, false, false);
      const uint32_t idesc_pv = idesc_bf16(128, 128, false, true);
      const uint32_t q0 = smem_u32(sQ);
      bool ok = mbar_wait(&bar->q_full, 0, guard);
      auto issue_qk = [&](int j) -> bool {
        const int s = j % kFStages, sb = j & 1;
        if (!mbar_wait(&bar->kv_full[s], (j / kFStages) & 1, guard)) return false;
        // the score buffer held P of tile j-2: its P·V must have completed
        if (j >= 2 && !mbar_wait(&bar->pv_done[sb], ((j - 2) >> 1) & 1, guard)) return false;
        tc_fence_after();
        const uint32_t k0 = smem_u32(sKV + s * kFStageBytes);
        for (int i = 0; i < 3; ++i) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_bf16(tmem + kFTmemS + sb * kFN, smem_desc_sw128(q0 + i * kFSlab + kk * 32, 16, 1024),
                      smem_desc_sw128(k0 + i * kFSlab + kk * 32, 16, 1024), idesc_qk,
                      (i | kk) != 0);
        }
        umma_commit(&bar->s_full[sb]);
        return true;
      };
      if (ok && ntiles > 0) ok = issue_qk(0);
      for (int j = 0; j < ntiles && ok; ++j) {
        if (j + 1 < ntiles && !issue_qk(j + 1)) { ok = false; break; }
        const int s = j % kFStages, sb = j & 1;
        if (!mbar_wait(&bar->p_full[sb], (j >> 1) & 1, guard)) { ok = false; break; }
        tc_fence_after();
        const uint32_t v0 = smem_u32(sKV + s * kFStageBytes + 3 * kFSlab);
#pragma unroll
        for (int k = 0; k < kFN / 16; ++k)
          umma_bf16_tmem_a(tmem + kFTmemO, tmem + kFTmemS + sb * kFN + k * 8,
                           smem_desc_sw128(v0 + k * 2048, kFSlab, 1024), idesc_pv,
                           (j == 0 && k == 0) ? 0u : 1u);
        umma_commit(&bar->kv_empty[s]);
        umma_commit(&bar->pv_done[sb]);
      }
      umma_commit(&bar->drain);
    }
  } else {
    // ---------------------------------------------------------------- softmax, epilogue
    const int quad = warp & 3;
    const int lane = static_cast<int>(lane_id());
    const int r = quad * 32 + lane;                       // query row in the tile = TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const int t = t0 + r;
    const int pos = p.start_pos + min(t, p.T - 1);        // rows past the chunk mirror its end
    const float c2 = p.scale_log2;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < ntiles; ++j) {
      const int sb = j & 1;
      if (!warp_wait(&bar->s_full[sb], (j >> 1) & 1, guard)) { ok = false; break; }
      tc_fence_after();
      float sc[kFN];
#pragma unroll
      for (int c = 0; c < kFN / 32; ++c) {
        float (&part)[32] = *reinterpret_cast<float(*)[32]>(&sc[32 * c]);
        tmem_ld32(tmem + lane_off + kFTmemS + sb * kFN + 32 * c, part);
      }
      const int key0 = j * kFN;
      const int nvis = pos - key0 + 1;                    // keys of this tile the row sees
#pragma unroll
      for (int i = 0; i < kFN; ++i) sc[i] = i < nvis ? sc[i] : -INFINITY;
      float mx = -INFINITY;
#pragma unroll
      for (int i = 0; i < kFN; ++i) mx = fmaxf(mx, sc[i]);
      const float mt = mx * c2;
      const bool raise = mt > m_run + kFRescale;
      // O holds tiles up to j-1 relative to m_run: rescale it (the warp waits for their last
      // P·V; rows that do not raise scale by 1) before P of tile j is released
      if (j > 0 && __any_sync(0xffffffffu, raise)) {
        if (!warp_wait(&bar->pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1, guard)) { ok = false; break; }
        tc_fence_after();
        const float f = raise ? fast_exp2(m_run - mt) : 1.f;
#pragma unroll 1
        for (int c = 0; c < 128 / 16; ++c) {
          float v[16];
          const uint32_t a = tmem + lane_off + kFTmemO + c * 16;
          tmem_ld16(a, v);
#pragma unroll
          for (int i = 0; i < 16; ++i) v[i] *= f;
          tmem_st16(a, v);
        }
      }
      if (raise) {
        if (m_run != -INFINITY) l_run *= fast_exp2(m_run - mt);
        m_run = mt;
      }
      uint32_t pk[kFN / 2];
      float sum = 0.f;
#pragma unroll
      for (int i = 0; i < kFN / 2; ++i) {
        const float a = fast_exp2(fmaf(sc[2 * i], c2, -m_run));
        const float e = fast_exp2(fmaf(sc[2 * i + 1], c2, -m_run));
        sum += a + e;
        pk[i] = pack_bf16x2(a, e);
      }
      l_run += sum;
#pragma unroll
      for (int c = 0; c < kFN / 32; ++c) {
        const uint32_t (&part)[16] = *reinterpret_cast<const uint32_t(*)[16]>(&pk[16 * c]);
        tmem_st16_u32(tmem + lane_off + kFTmemS + sb * kFN + 16 * c, part);
      }
      tc_fence_before();
      mbar_arrive(&bar->p_full[sb]);
    }
    if (ok && ntiles > 0) {
      const int jl = ntiles - 1;
      if (warp_wait(&bar->pv_done[jl & 1], (jl >> 1) & 1, guard)) {
        tc_fence_after();
        const float inv_l = 1.f / l_run;
        const bool live = t < p.T;
        uint4* dst = reinterpret_cast<uint4*>(
            p.out + (static_cast<size_t>(row0 + r) * p.n_heads + h) * kDv);
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          float v[32];
          tmem_ld32(tmem + lane_off + kFTmemO + 32 * c, v);
          uint32_t w[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) w[i] = pack_bf16x2(v[2 * i] * inv_l, v[2 * i + 1] * inv_l);
          if (live) {
#pragma unroll
            for (int q = 0; q < 4; ++q)
              dst[4 * c + q] = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
          }
        }
        if (live && p.lse)
          p.lse[static_cast<size_t>(row0 + r) * p.n_heads + h] =
              (m_run + log2f(l_run)) * 0.69314718055994531f;
      }
    }
  }

  // ------------------------------------------------------------------ teardown
  if (warp == 1) {
    int dummy = 0;
    Guard drain{reinterpret_cast<volatile int*>(&dummy), p.status};
    mbar_wait(&bar->drain, 0, drain);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

cudaError_t fmha_prepare() {
  return cudaFuncSetAttribute(fmha_prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              kFmhaSmem);
}

cudaError_t launch_fmha(const FmhaMaps& m, const FmhaParams& p, cudaStream_t s, bool pdl) {
  LaunchCfg lc(dim3((p.T + 127) / 128, p.n_heads, p.B), dim3(kFThreads), kFmhaSmem, s, pdl);
  return cudaLaunchKernelEx(&lc.cfg, fmha_prefill_kernel, m.qn, m.qp, m.kvb, m.pe, p);
}

}  // namespace mla
