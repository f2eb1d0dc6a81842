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
//   warps 2-..  epilogue, four warps per TMEM lane quadrant (warp % 4) splitting the 16-token
//               blocks (two in the merge and FP8 modes, which need the registers): tcgen05.ld
//               the fp32 accumulator (thread = weight row), apply RoPE for
//               the rotary rows of wq_b (partner of a pair = neighbouring lane), transpose 16
//               tokens at a time through shared memory and store bf16 as 16-byte vectors (8
//               consecutive rows of one token), hand the accumulator back — overlapping the next
//               unit's MMAs.
#include <cuda_fp8.h>

#include "internal.h"
#include "tc100.cuh"

namespace mla {

namespace {

// Epilogue warps: the epilogue of a 128 x 256 tile is a chain of 16-token blocks per warp
// (tcgen05.ld, transpose through shared memory, 16-byte stores) and paces large-N GEMMs, so the
// plain bf16 kernel runs four warps per TMEM lane quadrant.  The merge and FP8 modes keep two
// (their B builder and converters need the registers of a smaller block).
constexpr int kEpiWarps = 8;                            // merge / FP8 modes
constexpr int kEpiThreads = 32 * kEpiWarps;
template <bool FP8, bool MERGE>
__host__ __device__ constexpr int epi_warps() { return (FP8 || MERGE) ? kEpiWarps : 2 * kEpiWarps; }
// FP8: converter threads — four warps; two in the merge mode, whose B builder needs the registers
// (a block of more than 384 threads is held to 128 registers a thread)
template <bool MERGE>
__host__ __device__ constexpr int conv_threads() { return MERGE ? 64 : 128; }
constexpr int kSlabA = 128 * 64 * 2;   // 16 KB
constexpr int kSlabA8 = 128 * 64;      // 8 KB: an FP8 weight slab (64-byte rows, no swizzle)

template <bool FP8, bool MERGE = false>
constexpr int gemm_threads() { return 64 + 32 * epi_warps<FP8, MERGE>() + (FP8 ? conv_threads<MERGE>() : 0); }

template <int BN>
struct GemmTile {
  static constexpr int kSlabB = BN * 64 * 2;
  static constexpr int kTmemCols = 2 * BN < 32 ? 32 : 2 * BN;   // two accumulators
};

// MERGE (W_UV, K = 512): the ring carries only weight slabs; B (the token rows of o_lat, 8 K-slabs)
// is built once per output tile in a fixed region by the epilogue warps.
constexpr int kMergeSlabs = kC / 64;

// Plain-store epilogue: each epilogue warp transposes its 32 rows x 16 tokens of bf16 through a
// 1 KB staging block so that the global writes are 16-byte vectors.
constexpr int kEpiWarpStage = 32 * 16 * 2;

template <int BN, int STAGES, bool MERGE = false, bool FP8 = false>
constexpr int gemm_smem_bytes() {
  return 1024 /*align slack*/ + STAGES * kSlabA +
         (MERGE ? kMergeSlabs * GemmTile<BN>::kSlabB : STAGES * GemmTile<BN>::kSlabB) +
         (FP8 ? STAGES * kSlabA8 : 0) + 512 /*barriers*/ + epi_warps<FP8, MERGE>() * kEpiWarpStage;
}

// 16 FP8 E4M3 codes (bytes of v, lowest first) times `scale` → 16 bf16 (lo: codes 0-7).
// E4M3 values are exact in fp16 and fp32; the scaled value is rounded to fp32, then to bf16.
__device__ __forceinline__ void fp8x16_to_bf16(const uint4 v, float scale, uint4& lo, uint4& hi) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t o[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __half2 h0(__nv_cvt_fp8x2_to_halfraw2(
        static_cast<__nv_fp8x2_storage_t>(w[i] & 0xFFFFu), __NV_E4M3));
    const __half2 h1(__nv_cvt_fp8x2_to_halfraw2(
        static_cast<__nv_fp8x2_storage_t>(w[i] >> 16), __NV_E4M3));
    const float2 f0 = __half22float2(h0), f1 = __half22float2(h1);
    o[2 * i] = pack_bf16x2(f0.x * scale, f0.y * scale);
    o[2 * i + 1] = pack_bf16x2(f1.x * scale, f1.y * scale);
  }
  lo = make_uint4(o[0], o[1], o[2], o[3]);
  hi = make_uint4(o[4], o[5], o[6], o[7]);
}

// Builds B = o_lat[n0 .. n0+BN)[g][0..512) (bf16, K-major, 128-byte swizzle, 8 slabs of BN rows x
// 64 columns) for head g in shared memory, merging each row's split-K pieces by log-sum-exp
// weights; merged rows are also written to o_lat (and their lse to lse_out).  The epilogue warps
// (kEpiWarps) share the rows: warp w takes rows w, w+kEpiWarps, ... two at a time with all their
// loads in flight (the merge is a chain of dependent steps per row, so more warps hide more);
// lane l owns columns 16l .. 16l+15.  The tile's per-row piece records are read once (one per
// lane) and handed around by shuffles.
template <int BN>
__device__ void build_merged_b(const GemmParams& p, int g, int n0, uint8_t* sBm, int etid) {
  const int w = etid >> 5, lane = etid & 31;
  const int slab = lane >> 2, c0 = (lane & 3) * 2;   // this lane's 16 columns: slab, first chunk
  constexpr int kPieces = 3;                          // pieces of a row loaded per batch
  constexpr int kPre = (BN + 31) / 32;                // row records per lane
  int2 pre[kPre];                                     // row_pieces of the tile's rows
#pragma unroll
  for (int k = 0; k < kPre; ++k) {
    const int n = n0 + lane + 32 * k;
    pre[k] = n < p.N ? __ldcg(p.row_pieces + n) : make_int2(0, 0);
    // a record the key prefix cannot produce is reported and read as "one piece"
    const int lo = pre[k].x >> 1, hi = pre[k].y;
    if (n < p.N && (lo < 0 || hi < lo || hi >= p.n_pairs)) {
      atomicCAS(p.status, kDevOk, kDevBadArg);
      pre[k] = make_int2(0, 0);
    }
  }
  auto pieces_of = [&](int i) -> int2 {   // row_pieces[n0 + i], 0 <= i < BN (warp-uniform i)
    int2 v = make_int2(0, 0);
#pragma unroll
    for (int k = 0; k < kPre; ++k) {
      const int x = __shfl_sync(0xffffffffu, pre[k].x, i & 31);
      const int y = __shfl_sync(0xffffffffu, pre[k].y, i & 31);
      if ((i >> 5) == k) v = make_int2(x, y);
    }
    return v;
  };
#pragma unroll 1
  for (int i0 = w; i0 < BN; i0 += 2 * kEpiWarps) {
    int plo[2], phi[2], nn[2], slot_lo[2];
    float lse[2][kPieces];
    uint4 v[2][kPieces][2];
    // issue every load of both rows (o_lat row, or up to kPieces partial pieces) first
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int i = i0 + kEpiWarps * r;
      nn[r] = n0 + i;
      plo[r] = 0;
      phi[r] = -1;
      const int2 pcs = pieces_of(i < BN ? i : 0);
      if (i < BN && nn[r] < p.N) {
        plo[r] = pcs.x >> 1;
        slot_lo[r] = pcs.x & 1;   // the first piece is the tail of a pair begun in an earlier row
        phi[r] = pcs.y;
        const size_t orow = (static_cast<size_t>(nn[r]) * p.n_heads + g) * kC + lane * 16;
#pragma unroll
        for (int b = 0; b < kPieces; ++b) {
          const int q = plo[r] + b;
          lse[r][b] = -INFINITY;
          if (plo[r] == phi[r]) {
            if (b == 0) {   // one piece: the attention kernel wrote this row of o_lat
              const uint4* src = reinterpret_cast<const uint4*>(p.o_lat + orow);
              v[r][0][0] = src[0];
              v[r][0][1] = src[1];
            }
          } else if (q <= phi[r]) {
            const int slot = b == 0 ? slot_lo[r] : 0;
            const size_t base = (static_cast<size_t>(q) * 2 + slot) * 128 + g;
            lse[r][b] = p.part_lse[base];
            const uint4* src = reinterpret_cast<const uint4*>(p.part_o + base * kC + lane * 16);
            v[r][b][0] = src[0];
            v[r][b][1] = src[1];
          }
        }
      }
    }
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int i = i0 + kEpiWarps * r;
      if (i >= BN) continue;
      uint4 out_lo = make_uint4(0, 0, 0, 0), out_hi = make_uint4(0, 0, 0, 0);
      if (nn[r] < p.N) {
        if (plo[r] == phi[r]) {
          out_lo = v[r][0][0];
          out_hi = v[r][0][1];
        } else {
          // online log-sum-exp merge; rows of more than kPieces pieces load the rest here
          float mx = -INFINITY, wsum = 0.f, acc[16];
#pragma unroll
          for (int k = 0; k < 16; ++k) acc[k] = 0.f;
          for (int q0 = plo[r]; q0 <= phi[r]; q0 += kPieces) {
            float l_b[kPieces];
            uint4 v_b[kPieces][2];
#pragma unroll
            for (int b = 0; b < kPieces; ++b) {
              if (q0 == plo[r]) {
                l_b[b] = lse[r][b];
                v_b[b][0] = v[r][b][0];
                v_b[b][1] = v[r][b][1];
              } else {
                const int q = q0 + b;
                l_b[b] = -INFINITY;
                if (q <= phi[r]) {
                  const size_t base = static_cast<size_t>(q) * 2 * 128 + g;   // slot 0
                  l_b[b] = p.part_lse[base];
                  const uint4* src =
                      reinterpret_cast<const uint4*>(p.part_o + base * kC + lane * 16);
                  v_b[b][0] = src[0];
                  v_b[b][1] = src[1];
                }
              }
            }
            float m_new = mx;
#pragma unroll
            for (int b = 0; b < kPieces; ++b) m_new = fmaxf(m_new, l_b[b]);
            const float f = mx == -INFINITY ? 0.f : exp2f((mx - m_new) * 1.4426950408889634f);
            wsum *= f;
#pragma unroll
            for (int k = 0; k < 16; ++k) acc[k] *= f;
#pragma unroll
            for (int b = 0; b < kPieces; ++b) {
              if (q0 + b <= phi[r]) {
                const float wt = exp2f((l_b[b] - m_new) * 1.4426950408889634f);
                wsum += wt;
                const __half2* hv = reinterpret_cast<const __half2*>(v_b[b]);
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                  const float2 x = __half22float2(hv[k]);
                  acc[2 * k] = fmaf(wt, x.x, acc[2 * k]);
                  acc[2 * k + 1] = fmaf(wt, x.y, acc[2 * k + 1]);
                }
              }
            }
            mx = m_new;
          }
          const float inv = 1.f / wsum;
          uint32_t o[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) o[k] = pack_bf16x2(acc[2 * k] * inv, acc[2 * k + 1] * inv);
          out_lo = make_uint4(o[0], o[1], o[2], o[3]);
          out_hi = make_uint4(o[4], o[5], o[6], o[7]);
          uint4* dst = reinterpret_cast<uint4*>(
              p.o_lat + (static_cast<size_t>(nn[r]) * p.n_heads + g) * kC + lane * 16);
          dst[0] = out_lo;
          dst[1] = out_hi;
          if (lane == 0 && p.lse_out)
            p.lse_out[static_cast<size_t>(nn[r]) * p.n_heads + g] = mx + logf(wsum);
        }
      }
      uint8_t* rowp = sBm + slab * GemmTile<BN>::kSlabB + i * 128;
      *reinterpret_cast<uint4*>(rowp + ((c0 ^ (i & 7)) << 4)) = out_lo;
      *reinterpret_cast<uint4*>(rowp + (((c0 + 1) ^ (i & 7)) << 4)) = out_hi;
    }
  }
}

// The rotary (cos, sin) of row m's pair for tokens n0 .. n0+15, all loads issued before any
// store of the block (a store between them would keep each load waiting for the one before).
__device__ __forceinline__ void rope_prefetch(const GemmParams& p, int m, int n0, float2 (&cs)[16]) {
  const int h = m / kDq, j = m - h * kDq;
  if (p.epi != kEpiWqbRope || j < kDn) {
#pragma unroll
    for (int i = 0; i < 16; ++i) cs[i] = make_float2(1.f, 0.f);   // unused outside the rope rows
    return;
  }
  const int pair = (j - kDn) >> 1;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int n = n0 + i < p.N ? n0 + i : p.N - 1;
    cs[i] = __ldg(p.rope_tab + static_cast<size_t>(n) * kRopePairs + pair);
  }
}

// The value the epilogue stores for accumulator row m: the accumulator itself, or for the rotary
// rows of wq_b the rotated pair ("Query heads" mla-queries: q is a bf16 tensor before the
// rotation, so both inputs are rounded to bf16 first).
__device__ __forceinline__ float epi_value(const GemmParams& p, int m, float v, float partner,
                                           float2 cs) {
  if (p.epi == kEpiWqbRope) {
    const int j = m % kDq;
    if (j >= kDn) {
      v = bf16_round(v);
      partner = bf16_round(partner);
      return ((j - kDn) & 1) == 0 ? v * cs.x - partner * cs.y : partner * cs.y + v * cs.x;
    }
  }
  return v;
}

// Destination of the 8 consecutive accumulator rows m8 .. m8+7 (m8 a multiple of 8) for token n:
// 8 consecutive elements, since heads (192 rows) and their content part (128) are multiples of 8.
__device__ __forceinline__ bf16* epi_dst8(const GemmParams& p, int g, int m8, int n) {
  if (p.epi == kEpiWqbRope) {
    const int h = m8 / kDq, j = m8 - h * kDq;
    if (j < kDn) return p.out0 + static_cast<size_t>(n) * p.ld_n0 + static_cast<size_t>(h) * kDn + j;
    return p.out1 + (static_cast<size_t>(n) * kHPad + h) * kDk + kC + (j - kDn);
  }
  return p.out0 + static_cast<size_t>(n) * p.ld_n0 + static_cast<size_t>(g) * p.ld_g0 + m8;
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

// Work split: CTA c takes output tiles c, c + G, c + 2G, ... (G = grid size).
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

template <int BN, int STAGES, bool MERGE, bool FP8>
__global__ void __launch_bounds__(gemm_threads<FP8, MERGE>(), 1)
    gemm_bf16_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const GemmParams p, const int batches) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sA = smem;                      // bf16 weight slabs (FP8: written by the converters)
  uint8_t* sB = smem + STAGES * kSlabA;   // MERGE: the tile's 8 B slabs; else the ring's B slabs
  constexpr int kSmemB = MERGE ? kMergeSlabs * GemmTile<BN>::kSlabB : STAGES * GemmTile<BN>::kSlabB;
  uint8_t* sA8 = sB + kSmemB;              // FP8: the ring's fp8 weight slabs
  constexpr uint32_t kStageTx =
      (FP8 ? kSlabA8 : kSlabA) + (MERGE ? 0 : GemmTile<BN>::kSlabB);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sA8 + (FP8 ? STAGES * kSlabA8 : 0));
  uint64_t* full = bars;
  uint64_t* empty = bars + STAGES;
  uint64_t* acc_full = bars + 2 * STAGES;        // [2]
  uint64_t* acc_empty = bars + 2 * STAGES + 2;   // [2]
  uint64_t* drain = bars + 2 * STAGES + 4;
  uint64_t* b_ready = bars + 2 * STAGES + 5;     // MERGE: the tile's B block is built
  uint64_t* conv = bars + 2 * STAGES + 6;        // FP8: [STAGES] the slab is converted
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 3 * STAGES + 6);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  uint8_t* sEpi = reinterpret_cast<uint8_t*>(bars) + 512;   // plain-store epilogue staging
  static_assert((3 * 10 + 6) * 8 + 8 <= 512, "barrier block");

  pdl_launch_dependents();
  const int warp = warp_id();
  const int nk = p.K / 64;
  const int mt = (p.M + 127) / 128;   // a last partial tile reads zero rows (TMA fill)
  const int nt = (p.N + BN - 1) / BN;
  const int total = batches * mt * nt;
  Guard guard{abort_flag, p.status, p.wait_limit_ns ? p.wait_limit_ns : kWaitLimitNs};
  Sched sched;
  sched.init(total, gridDim.x, blockIdx.x);

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 32 * epi_warps<FP8, MERGE>());
    }
    mbar_init(drain, 1);
    mbar_init(b_ready, kEpiThreads);
    if (FP8)
      for (int i = 0; i < STAGES; ++i) mbar_init(&conv[i], conv_threads<MERGE>());
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
  int issued = 0;   // producer thread: ring slots whose loads it issued

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
            mbar_arrive_expect_tx(&full[npre], kStageTx);
            tma_load_3d_hint(FP8 ? sA8 + npre * kSlabA8 : sA + npre * kSlabA, &tmA, &full[npre],
                             j * 64, un.m0 + p.a_row_off, un.g, pol_w);
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
            mbar_arrive_expect_tx(&full[s], kStageTx);
            tma_load_3d_hint(FP8 ? sA8 + s * kSlabA8 : sA + s * kSlabA, &tmA, &full[s], j * 64,
                             un.m0 + p.a_row_off, un.g, pol_w);
          }
          if (!MERGE)
            tma_load_3d(sB + s * GemmTile<BN>::kSlabB, &tmB, &full[s], j * 64, p.b_g0 ? 0 : un.g,
                        un.n0);
        }
      }
      issued = ks;   // slots [0, ks) were armed and loaded (a failed slot breaks before)
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
        if (MERGE && !mbar_wait(b_ready, si & 1, guard)) break;
        tc_fence_after();
        const uint32_t d = tmem + ab * BN;
        for (int j = 0; j < nk; ++j, ++ks) {
          const int s = ks % STAGES;
          if (!mbar_wait(FP8 ? &conv[s] : &full[s], (ks / STAGES) & 1, guard)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + s * kSlabA);
          const uint32_t b0 = smem_u32(sB + (MERGE ? j : s) * GemmTile<BN>::kSlabB);
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
  } else if (FP8 && warp >= 2 + epi_warps<FP8, MERGE>()) {
    // FP8 converter warps: each ring slab of fp8 weight codes → bf16 (code × the block's scale)
    // in the 128-byte-swizzled layout the MMA reads; thread t converts 16-byte chunks t, t + T,
    // t + 2T, ... of the slab (T converter threads; row = chunk / 4, 16 columns each).  A slab (128 rows x 64
    // columns) lies in one 128 x 128 scale block.  Lane b of every converter warp holds the scale
    // of K block b of the current tile and has the next tile's in flight, so no slab waits on a
    // scale load (the launcher limits FP8 GEMMs to K <= 32 * 128).
    const int ctid = static_cast<int>(threadIdx.x) - (64 + 32 * epi_warps<FP8, MERGE>());
    const int lane = static_cast<int>(lane_id());
    const int kblocks = (p.K + 127) / 128;
    auto tile_scale = [&](int unit) -> float {   // this lane's K block of tile `unit`
      if (unit < 0 || lane >= kblocks) return 0.f;
      const Unit un = unit_of(unit, mt, nt, BN);
      const long long si = un.g * p.a_sg + ((un.m0 + p.a_row_off) >> 7) * p.a_sm + lane * p.a_sk;
      if (si >= 0 && si < p.a_scale_n) return __ldg(p.a_scale + si);
      guard.fail(kDevBadArg);   // a scale index outside the tensor: reported, not read
      return 0.f;
    };
    int ks = 0;
    int u;
    bool ok = true;
    Sched ahead = sched;   // one tile ahead of `sched`
    int u_next = -1;
    float sc_next = 0.f;
    if (ahead.next(u_next)) sc_next = tile_scale(u_next);
    while (ok && sched.next(u)) {
      const float sc_cur = sc_next;   // tile u's scales (u == u_next)
      u_next = -1;
      sc_next = ahead.next(u_next) ? tile_scale(u_next) : 0.f;
      for (int j = 0; j < nk; ++j, ++ks) {
        const int s = ks % STAGES;
        const float scale = __shfl_sync(0xffffffffu, sc_cur, (j * 64) >> 7);
        // voted wait: the warp stays converged for the next shuffle
        if (!warp_wait(&full[s], (ks / STAGES) & 1, guard)) { ok = false; break; }
        const uint8_t* src = sA8 + s * kSlabA8;
        uint8_t* dst = sA + s * kSlabA;
#pragma unroll
        for (int q = 0; q < 512 / conv_threads<MERGE>(); ++q) {   // 512 chunks of 16 bytes
          const int ch = ctid + conv_threads<MERGE>() * q;
          const int r = ch >> 2, c = ch & 3;
          const uint4 v = *reinterpret_cast<const uint4*>(src + r * 64 + c * 16);
          uint4 lo, hi;
          fp8x16_to_bf16(v, scale, lo, hi);
          *reinterpret_cast<uint4*>(dst + r * 128 + (((2 * c) ^ (r & 7)) << 4)) = lo;
          *reinterpret_cast<uint4*>(dst + r * 128 + (((2 * c + 1) ^ (r & 7)) << 4)) = hi;
        }
        fence_async_smem();   // generic-proxy writes → visible to the tensor core
        mbar_arrive(&conv[s]);
      }
    }
  } else {
    // epilogue warps 2 .. 1 + epi_warps → TMEM lane quadrant warp % 4
    pdl_wait();   // outputs may be read by the kernel before this one
    const int quad = warp & 3;
    const int row = quad * 32 + static_cast<int>(lane_id());
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const int etid = static_cast<int>(threadIdx.x) - 64;   // 0 .. 32 * epi_warps - 1
    constexpr int kSub = epi_warps<FP8, MERGE>() / 4;       // warps per lane quadrant
    const int sub = etid >> 7;    // the warps of a lane quadrant split the 16-token blocks
    // the epilogue writes 16-byte vectors: every 8-row group must start 16-byte aligned (the C
    // ABI requires aligned outputs; a violation is reported, never written)
    const bool aligned_out =
        (reinterpret_cast<uintptr_t>(p.out0) & 15) == 0 && (p.ld_n0 & 7) == 0 &&
        (p.epi == kEpiStore ? (p.ld_g0 & 7) == 0
                            : (reinterpret_cast<uintptr_t>(p.out1) & 15) == 0);
    if (!aligned_out && etid == 0) guard.fail(kDevBadArg);
    int si = 0;
    int u;
    while (sched.next(u)) {
      const Unit un = unit_of(u, mt, nt, BN);
      const int ab = si & 1;
      if constexpr (MERGE) {
        // the previous tile's MMAs have completed (its acc_full was observed): rebuild B
        build_merged_b<BN>(p, un.g, un.n0, sB, etid);
        fence_async_smem();
        mbar_arrive(b_ready);
      }
      if (!warp_wait(&acc_full[ab], (si >> 1) & 1, guard)) break;
      tc_fence_after();
      const int m = un.m0 + row;
      if (!aligned_out) break;
      // 16-token blocks: lane = row, value i = token; bf16 into this warp's staging block as
      // [token][32 rows], then each lane writes two 16-byte pieces (8 rows of one token)
      __nv_bfloat16* stg = reinterpret_cast<__nv_bfloat16*>(sEpi + (warp - 2) * 1024);
      const int mw = un.m0 + quad * 32;   // first row of this warp
      const bool rope_epi = p.epi == kEpiWqbRope;   // only the rotary rows need the partner row
#pragma unroll 1
      for (int c0 = 16 * sub; c0 < BN; c0 += 16 * kSub) {
        if (un.n0 + c0 >= p.N) break;   // uniform across the warp
        float v[16];
        float2 cs[16];
        rope_prefetch(p, m, un.n0 + c0, cs);
        tmem_ld16(tmem + lane_off + ab * BN + c0, v);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float partner = rope_epi ? __shfl_xor_sync(0xffffffffu, v[i], 1) : 0.f;
          stg[i * 32 + lane_id()] = __float2bfloat16_rn(epi_value(p, m, v[i], partner, cs[i]));
        }
        __syncwarp();
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int c = static_cast<int>(lane_id()) + 32 * j;   // 64 pieces of 16 bytes
          const int t = c >> 2, part = c & 3;
          const int n = un.n0 + c0 + t;
          if (n < p.N && mw + part * 8 < p.M)   // M is a multiple of 8: whole groups only
            *reinterpret_cast<uint4*>(epi_dst8(p, un.g, mw + part * 8, n)) =
                *reinterpret_cast<const uint4*>(stg + t * 32 + part * 8);
        }
        __syncwarp();   // the block is read before the next one overwrites it
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[ab]);
      ++si;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (issued > 0 && guard.aborted()) {
    // a role gave up (possibly after the producer had issued everything): the ring's last loads
    // may still be in flight, so they land before the CTA's shared memory goes away
    int dummy = 0;
    Guard dr{reinterpret_cast<volatile int*>(&dummy), p.status};
    for (int k = issued > STAGES ? issued - STAGES : 0; k < issued; ++k)
      mbar_wait(&full[k % STAGES], (k / STAGES) & 1, dr);
  }
  if (warp == 1) {
    int dummy = 0;
    Guard dr{reinterpret_cast<volatile int*>(&dummy), p.status};
    mbar_wait(drain, 0, dr);   // no MMA still writes the accumulators
    tc_fence_after();
    tmem_dealloc(tmem, GemmTile<BN>::kTmemCols);
  }
}

int g_num_sms = 0;

template <int BN, int STAGES, bool MERGE, bool FP8 = false>
cudaError_t launch_gemm_t(const CUtensorMap& ta, const CUtensorMap& tb, const GemmParams& p,
                          int batches, cudaStream_t s, bool pdl) {
  if (g_num_sms == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&g_num_sms, cudaDevAttrMultiProcessorCount, dev);
    if (g_num_sms <= 0) g_num_sms = 1;
  }
  const int total = batches * ((p.M + 127) / 128) * ((p.N + BN - 1) / BN);
  const int grid = total < g_num_sms ? total : g_num_sms;
  LaunchCfg lc(dim3(grid), dim3(gemm_threads<FP8, MERGE>()), gemm_smem_bytes<BN, STAGES, MERGE, FP8>(), s,
               pdl);
  return cudaLaunchKernelEx(&lc.cfg, gemm_bf16_kernel<BN, STAGES, MERGE, FP8>, ta, tb, p, batches);
}

template <int BN, int STAGES, bool MERGE, bool FP8 = false>
cudaError_t set_attr() {
  static_assert(gemm_smem_bytes<BN, STAGES, MERGE, FP8>() <= 232448, "shared memory budget");
  return cudaFuncSetAttribute(gemm_bf16_kernel<BN, STAGES, MERGE, FP8>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize,
                              gemm_smem_bytes<BN, STAGES, MERGE, FP8>());
}

}  // namespace

// Tile choice: BN covers the token count up to 256; the ring fills ~200 KB of shared memory.
// The merge mode (W_UV for at most 64 rows) keeps 8 B slabs resident and a 10/8-stage A ring.
cudaError_t launch_gemm(const CUtensorMap& ta, const CUtensorMap& tb, const GemmParams& p,
                        int batches, cudaStream_t s, bool pdl) {
  if (p.a_scale) {   // FP8 weights: an 8 KB fp8 slab per stage on top of the bf16 one
    if (p.K > 32 * 128) return cudaErrorInvalidValue;   // one scale per lane of a warp
    if (p.bmerge) {
      if (p.K != kC || p.N > 64) return cudaErrorInvalidValue;
      if (p.N <= 32) return launch_gemm_t<32, 7, true, true>(ta, tb, p, batches, s, pdl);
      return launch_gemm_t<64, 6, true, true>(ta, tb, p, batches, s, pdl);
    }
    if (p.N <= 32) return launch_gemm_t<32, 7, false, true>(ta, tb, p, batches, s, pdl);
    if (p.N <= 64) return launch_gemm_t<64, 6, false, true>(ta, tb, p, batches, s, pdl);
    if (p.N <= 128) return launch_gemm_t<128, 5, false, true>(ta, tb, p, batches, s, pdl);
    return launch_gemm_t<256, 3, false, true>(ta, tb, p, batches, s, pdl);
  }
  if (p.bmerge) {
    if (p.K != kC || p.N > 64) return cudaErrorInvalidValue;
    if (p.N <= 32) return launch_gemm_t<32, 10, true>(ta, tb, p, batches, s, pdl);
    return launch_gemm_t<64, 8, true>(ta, tb, p, batches, s, pdl);
  }
  if (p.N <= 32) return launch_gemm_t<32, 10, false>(ta, tb, p, batches, s, pdl);
  if (p.N <= 64) return launch_gemm_t<64, 8, false>(ta, tb, p, batches, s, pdl);
  if (p.N <= 128) return launch_gemm_t<128, 6, false>(ta, tb, p, batches, s, pdl);
  return launch_gemm_t<256, 4, false>(ta, tb, p, batches, s, pdl);
}

cudaError_t gemm_prepare() {
  cudaError_t e;
  if ((e = set_attr<32, 10, false>()) != cudaSuccess) return e;
  if ((e = set_attr<64, 8, false>()) != cudaSuccess) return e;
  if ((e = set_attr<128, 6, false>()) != cudaSuccess) return e;
  if ((e = set_attr<256, 4, false>()) != cudaSuccess) return e;
  if ((e = set_attr<32, 10, true>()) != cudaSuccess) return e;
  if ((e = set_attr<64, 8, true>()) != cudaSuccess) return e;
  if ((e = set_attr<32, 7, false, true>()) != cudaSuccess) return e;
  if ((e = set_attr<64, 6, false, true>()) != cudaSuccess) return e;
  if ((e = set_attr<128, 5, false, true>()) != cudaSuccess) return e;
  if ((e = set_attr<256, 3, false, true>()) != cudaSuccess) return e;
  if ((e = set_attr<32, 7, true, true>()) != cudaSuccess) return e;
  return set_attr<64, 6, true, true>();
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

// FP8 codes of W_UK^T: w_ukt[h][c][d] = wkv_b[h*256 + d][c] (bytes), d < 128.
__global__ void transpose_uk_fp8_kernel(const uint8_t* __restrict__ wkv_b,
                                        uint8_t* __restrict__ w_ukt) {
  __shared__ uint8_t tile[32][33];
  const int h = blockIdx.z;
  const int c0 = blockIdx.x * 32, d0 = blockIdx.y * 32;
  const int tx = threadIdx.x, ty = threadIdx.y;   // 32 x 8
  for (int i = ty; i < 32; i += 8)
    tile[i][tx] = wkv_b[(static_cast<size_t>(h) * (kDn + kDv) + d0 + i) * kC + c0 + tx];
  __syncthreads();
  for (int i = ty; i < 32; i += 8)
    w_ukt[(static_cast<size_t>(h) * kC + c0 + i) * kDn + d0 + tx] = tile[tx][i];
}

cudaError_t launch_transpose_uk_fp8(const uint8_t* wkv_b, uint8_t* w_ukt, int n_heads,
                                    cudaStream_t s) {
  dim3 grid(kC / 32, kDn / 32, n_heads), block(32, 8);
  transpose_uk_fp8_kernel<<<grid, block, 0, s>>>(wkv_b, w_ukt);
  return cudaGetLastError();
}

cudaError_t launch_transpose_uk(const bf16* wkv_b, bf16* w_ukt, int n_heads, cudaStream_t s) {
  dim3 grid(kC / 32, kDn / 32, n_heads), block(32, 8);
  transpose_uk_kernel<<<grid, block, 0, s>>>(wkv_b, w_ukt);
  return cudaGetLastError();
}

}  // namespace mla
