// k_attn.cu — a5–a7: latent scores, fp32 softmax and the weighted sum over cached latents.
//
// "DeepSeek-V3.2-Exp · Attention update", mla-decode excerpt:
//   scores[h, t] = (q_lat[h] · kv_cache[t] + q_pe[h] · pe_cache[t]) * softmax_scale,
//   p = softmax_t(scores) (fp32),  o_lat[h] = sum_t p[h, t] · kv_cache[t].
// "Kimi-K2 · value_states", mla-prefill excerpt: a prefill chunk adds the causal mask (key t is
// visible to query i iff t <= position of i).
//
// Design (B200):
//   * One query row (one token of one sequence) at a time; its heads form the MMA M dimension
//     (128 rows, heads beyond H are zero rows), so QK^T and P·V are dense 128-row tcgen05 MMAs.
//   * A cluster of TWO CTAs (one SM each) handles a row.  CTA 0 owns the latent columns
//     [0, 256), CTA 1 owns [256, 512) plus the 64 rotary columns.  Each CTA loads only its
//     columns of every cache tile (so the 576-wide cache row is read from HBM once), computes a
//     partial score tile over its columns, and the two partials are exchanged through
//     distributed shared memory; both CTAs then hold identical full scores and run the identical
//     online softmax.  Each CTA accumulates the value half it owns: O[128 x 256] fp32 in TMEM
//     (256 columns), plus two 64-column score buffers.
//   * Keys are streamed in tiles of 64 by TMA (128-byte swizzle, evict-first), two stages deep.
//   * The flattened key range of all rows is split evenly over the cluster pairs (split-K over
//     keys, also across row boundaries); a row cut between pairs leaves normalised partials
//     (O/l, lse) for the combine kernel, an uncut row is written as bf16 o_lat directly.
//   * Online softmax in exp2 domain with lazy rescaling: the running max is only raised (and O
//     in TMEM rescaled) when a tile's max exceeds it by more than 8 (factor 256), which keeps the
//     rescale off the common path while the result stays exact.
//   * Warp roles: warp 0 TMA producer, warp 1 TMEM owner + MMA issuer, warps 2-5 softmax and
//     epilogue (thread = head row = TMEM lane).
#include "internal.h"
#include "tc100.cuh"

namespace mla {

namespace {

constexpr int kNK = 64;                    // keys per tile
constexpr int kStages = 2;                 // cache tile ring depth
constexpr int kSlabKV = kNK * 128;         // 8 KB: 64 columns x 64 keys, bf16
constexpr int kSlabQ = 128 * 128;          // 16 KB: 64 columns x 128 heads, bf16
constexpr int kMaxSlabs = 5;               // rank 1: 4 latent slabs + 1 rotary slab
constexpr int kStageBytes = kMaxSlabs * kSlabKV;
constexpr int kPBytes = 128 * kNK * 2;     // 16 KB
constexpr int kXBytes = 128 * kNK * 4;     // 32 KB

constexpr int kOffQ = 0;
constexpr int kOffKV = kOffQ + kMaxSlabs * kSlabQ;        // 80 KB
constexpr int kOffP = kOffKV + kStages * kStageBytes;     // 160 KB
constexpr int kOffX = kOffP + 2 * kPBytes;                // 192 KB
constexpr int kOffBar = kOffX + kXBytes;                  // 224 KB
constexpr int kAttnSmem = kOffBar + 256 + 1024;

constexpr int kTmemCols = 512;
constexpr uint32_t kTmemO = 0;             // columns [0, 256)
constexpr uint32_t kTmemS = 256;           // two 64-column score buffers

constexpr int kThreads = 192;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

struct Bars {
  uint64_t q_full, q_empty;
  uint64_t kv_full[kStages], kv_empty[kStages];
  uint64_t s_full[2], s_empty[2];
  uint64_t p_full[2], pv_done[2];
  uint64_t o_empty;
  uint64_t x_full, x_empty;
  uint64_t drain;
  uint32_t tmem_slot;
  int abort_flag;
};
static_assert(sizeof(Bars) <= 256, "barrier block");

// Row containing flattened key e: largest r with prefix[r] <= e.
__device__ __forceinline__ int row_of_key(const long long* prefix, int rows, long long e) {
  int lo = 0, hi = rows - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(prefix + mid) <= e) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

// Iterates the pieces (row, [k0, k1)) of one pair's key range.
struct PieceIter {
  const long long* prefix;
  int rows;
  long long e0, e1;
  int r;
  __device__ void init(const long long* pf, int nrows, long long b, long long e) {
    prefix = pf;
    rows = nrows;
    e0 = b;
    e1 = e;
    r = row_of_key(pf, nrows, b);
  }
  // Fills the current piece; false when the range is exhausted.
  __device__ bool get(int& row, int& k0, int& k1, int& nkeys_row, bool& first_row) const {
    if (r >= rows) return false;
    const long long R0 = __ldg(prefix + r), R1 = __ldg(prefix + r + 1);
    if (R0 >= e1) return false;
    row = r;
    k0 = static_cast<int>((e0 > R0 ? e0 : R0) - R0);
    k1 = static_cast<int>((e1 < R1 ? e1 : R1) - R0);
    nkeys_row = static_cast<int>(R1 - R0);
    first_row = (R0 <= e0);
    return true;
  }
  __device__ void next() { ++r; }
};

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    latent_attention_kernel(const __grid_constant__ CUtensorMap tmQ,
                            const __grid_constant__ CUtensorMap tmKV,
                            const __grid_constant__ CUtensorMap tmPE, const AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem + kOffQ;
  uint8_t* sKV = smem + kOffKV;
  uint8_t* sP = smem + kOffP;
  float* sX = reinterpret_cast<float*>(smem + kOffX);
  Bars* bar = reinterpret_cast<Bars*>(smem + kOffBar);

  const uint32_t rank = cluster_ctarank();
  const uint32_t peer = rank ^ 1u;
  const int pair = static_cast<int>(cluster_id_x());
  const int launched_pairs = static_cast<int>(nclusters_x());
  const long long total = __ldg(p.row_prefix + p.rows);
  const int pairs = active_pairs(total, launched_pairs, p.min_keys_per_pair);
  if (pair >= pairs) return;   // both CTAs of the pair take this branch together
  const long long e0 = pair_begin(total, pairs, pair), e1 = pair_begin(total, pairs, pair + 1);

  const int warp = static_cast<int>(warp_id());
  const int nslabs = rank == 0 ? 4 : 5;           // column slabs this CTA owns
  const int col0 = rank == 0 ? 0 : 256;           // first latent column
  Guard guard{reinterpret_cast<volatile int*>(&bar->abort_flag), p.status};

  if (threadIdx.x == 0) {
    mbar_init(&bar->q_full, 1);
    mbar_init(&bar->q_empty, 1);
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&bar->kv_full[i], 1);
      mbar_init(&bar->kv_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar->s_full[i], 1);
      mbar_init(&bar->s_empty[i], 128);
      mbar_init(&bar->p_full[i], 128);
      mbar_init(&bar->pv_done[i], 1);
    }
    mbar_init(&bar->o_empty, 128);
    mbar_init(&bar->x_full, 128);
    mbar_init(&bar->x_empty, 128);
    mbar_init(&bar->drain, 1);
    bar->abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmKV);
    tma_prefetch_desc(&tmPE);
  }
  if (warp == 1) tmem_alloc(&bar->tmem_slot, kTmemCols);
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();   // the peer's barriers are initialised before any remote arrive
  tc_fence_after();
  const uint32_t tmem = bar->tmem_slot;

  PieceIter it;
  it.init(p.row_prefix, p.rows, e0, e1);

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (elect_one()) {
      const uint64_t pol = policy_evict_first();
      int g = 0, piece = 0;
      int last_q = -1;
      int last_tile[kStages] = {-1, -1};
      int row, k0, k1, nrow;
      bool first_row;
      while (!guard.aborted() && it.get(row, k0, k1, nrow, first_row)) {
        const int b = row / p.T;
        if (piece > 0 && !mbar_wait(&bar->q_empty, (piece - 1) & 1, guard)) break;
        mbar_arrive_expect_tx(&bar->q_full, nslabs * kSlabQ);
        for (int i = 0; i < nslabs; ++i)
          tma_load_3d(sQ + i * kSlabQ, &tmQ, &bar->q_full, col0 + 64 * i, 0, row);
        last_q = piece;
        const int ntiles = (k1 - k0 + kNK - 1) / kNK;
        bool ok = true;
        for (int j = 0; j < ntiles; ++j, ++g) {
          const int s = g % kStages;
          if (g >= kStages && !mbar_wait(&bar->kv_empty[s], ((g / kStages) - 1) & 1, guard)) {
            ok = false;
            break;
          }
          uint64_t* fb = &bar->kv_full[s];
          mbar_arrive_expect_tx(fb, nslabs * kSlabKV);
          uint8_t* dst = sKV + s * kStageBytes;
          const int key = k0 + j * kNK;
          for (int i = 0; i < 4; ++i)
            tma_load_3d_hint(dst + i * kSlabKV, &tmKV, fb, col0 + 64 * i, key, b, pol);
          if (rank == 1) tma_load_3d_hint(dst + 4 * kSlabKV, &tmPE, fb, 0, key, b, pol);
          last_tile[s] = g;
        }
        if (!ok) break;
        ++piece;
        it.next();
      }
      if (guard.aborted()) {
        int dummy = 0;
        Guard drain{reinterpret_cast<volatile int*>(&dummy), p.status};
        if (last_q >= 0) mbar_wait(&bar->q_full, last_q & 1, drain);
        for (int s = 0; s < kStages; ++s)
          if (last_tile[s] >= 0) mbar_wait(&bar->kv_full[s], (last_tile[s] / kStages) & 1, drain);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (elect_one()) {
      const uint32_t idesc_qk = idesc_bf16(128, kNK, false, false);
      const uint32_t idesc_pv = idesc_bf16(128, 256, false, true);
      const uint32_t q_base = smem_u32(sQ);
      int g = 0, piece = 0;
      int row, k0, k1, nrow;
      bool first_row;
      // P·V for tile t (A = P buffer, K-major; B = the stage's latent slabs, MN-major)
      auto issue_pv = [&](int t, bool first, int pc) -> bool {
        const int pb = t & 1, s = t % kStages;
        if (!mbar_wait(&bar->p_full[pb], (t >> 1) & 1, guard)) return false;
        if (first && pc > 0 && !mbar_wait(&bar->o_empty, (pc - 1) & 1, guard)) return false;
        tc_fence_after();
        const uint32_t a0 = smem_u32(sP + pb * kPBytes);
        const uint32_t b0 = smem_u32(sKV + s * kStageBytes);
#pragma unroll
        for (int k = 0; k < kNK / 16; ++k) {
          umma_bf16(tmem + kTmemO, smem_desc_sw128(a0 + k * 32, 16, 1024),
                    smem_desc_sw128(b0 + k * 2048, kSlabKV, 1024), idesc_pv,
                    (first && k == 0) ? 0u : 1u);
        }
        umma_commit(&bar->kv_empty[s]);
        umma_commit(&bar->pv_done[pb]);
        return true;
      };
      bool ok = true;
      while (ok && it.get(row, k0, k1, nrow, first_row)) {
        const int ntiles = (k1 - k0 + kNK - 1) / kNK;
        if (!mbar_wait(&bar->q_full, piece & 1, guard)) break;
        for (int j = 0; j < ntiles && ok; ++j, ++g) {
          const int s = g % kStages, sb = g & 1;
          if (!mbar_wait(&bar->kv_full[s], (g / kStages) & 1, guard)) { ok = false; break; }
          if (g >= 2 && !mbar_wait(&bar->s_empty[sb], ((g >> 1) - 1) & 1, guard)) { ok = false; break; }
          tc_fence_after();
          const uint32_t kv0 = smem_u32(sKV + s * kStageBytes);
          for (int i = 0; i < nslabs; ++i) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              umma_bf16(tmem + kTmemS + sb * kNK,
                        smem_desc_sw128(q_base + i * kSlabQ + kk * 32, 16, 1024),
                        smem_desc_sw128(kv0 + i * kSlabKV + kk * 32, 16, 1024), idesc_qk,
                        (i | kk) != 0);
            }
          }
          umma_commit(&bar->s_full[sb]);
          if (j == ntiles - 1) umma_commit(&bar->q_empty);
          if (j > 0 && !issue_pv(g - 1, j - 1 == 0, piece)) { ok = false; break; }
        }
        if (!ok) break;
        if (!issue_pv(g - 1, ntiles == 1, piece)) break;
        ++piece;
        it.next();
      }
      umma_commit(&bar->drain);
    }
  } else {
    // ---------------------------------------------------------------- softmax + epilogue
    const int quad = warp & 3;
    const int h = quad * 32 + static_cast<int>(lane_id());   // head row = TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t x_remote = mapa_shared(smem_u32(sX), peer);
    const uint32_t xfull_remote = mapa_shared(smem_u32(&bar->x_full), peer);
    const uint32_t xempty_remote = mapa_shared(smem_u32(&bar->x_empty), peer);
    const int tid = static_cast<int>(threadIdx.x) - 64;     // 0..127
    int g = 0, piece = 0;
    int row, k0, k1, nrow;
    bool first_row;
    bool ok = true;
    while (ok && it.get(row, k0, k1, nrow, first_row)) {
      const int ntiles = (k1 - k0 + kNK - 1) / kNK;
      float m_run = -INFINITY, l_run = 0.f;
      for (int j = 0; j < ntiles; ++j, ++g) {
        const int sb = g & 1;
        if (!mbar_wait(&bar->s_full[sb], (g >> 1) & 1, guard)) { ok = false; break; }
        tc_fence_after();
        float s[kNK];
#pragma unroll
        for (int c = 0; c < kNK / 16; ++c) {
          float v[16];
          tmem_ld16(tmem + lane_off + kTmemS + sb * kNK + c * 16, v);
#pragma unroll
          for (int i = 0; i < 16; ++i) s[c * 16 + i] = v[i];
        }
        tc_fence_before();
        mbar_arrive(&bar->s_empty[sb]);

        // exchange the partial scores with the peer CTA
        if (g >= 1 && !mbar_wait<true>(&bar->x_empty, (g - 1) & 1, guard)) { ok = false; break; }
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const uint32_t off = static_cast<uint32_t>(h * 256 + (((c + h) & 15) << 4));
          st_cluster_v4(x_remote + off, s[4 * c], s[4 * c + 1], s[4 * c + 2], s[4 * c + 3]);
        }
        mbar_arrive_remote(xfull_remote);
        if (!mbar_wait<true>(&bar->x_full, g & 1, guard)) { ok = false; break; }
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const float4 x = *reinterpret_cast<const float4*>(
              reinterpret_cast<const uint8_t*>(sX) + h * 256 + (((c + h) & 15) << 4));
          s[4 * c] += x.x;
          s[4 * c + 1] += x.y;
          s[4 * c + 2] += x.z;
          s[4 * c + 3] += x.w;
        }
        mbar_arrive_remote(xempty_remote);

        // online softmax (log2 domain)
        const int key0 = k0 + j * kNK;
        const int nvalid = min(kNK, k1 - key0);
        float mt = -INFINITY;
#pragma unroll
        for (int i = 0; i < kNK; ++i) {
          const float x = i < nvalid ? s[i] * p.scale_log2 : -INFINITY;
          s[i] = x;
          mt = fmaxf(mt, x);
        }
        if (p.logits && rank == 0 && h < p.n_heads) {
          float* lg = p.logits + (static_cast<size_t>(row) * p.n_heads + h) * p.max_seq_len + key0;
          const float to_nat = p.scale / p.scale_log2;
#pragma unroll
          for (int i = 0; i < kNK; ++i)
            if (i < nvalid) lg[i] = s[i] * to_nat;
        }
        const float m_new = fmaxf(m_run, mt);
        if (m_new > m_run + kRescaleThreshold) {
          if (j > 0) {
            // O holds the earlier tiles: wait for their last P·V, then rescale the row in TMEM
            if (!mbar_wait(&bar->pv_done[(g - 1) & 1], ((g - 1) >> 1) & 1, guard)) { ok = false; break; }
            tc_fence_after();
            const float f = exp2f(m_run - m_new);
            l_run *= f;
#pragma unroll 1
            for (int c = 0; c < 256 / 16; ++c) {
              float v[16];
              tmem_ld16(tmem + lane_off + kTmemO + c * 16, v);
#pragma unroll
              for (int i = 0; i < 16; ++i) v[i] *= f;
              tmem_st16(tmem + lane_off + kTmemO + c * 16, v);
            }
          }
          m_run = m_new;
        }
        // P tile (bf16, K-major, 128-byte swizzle): row h, 16-byte chunk c at (c ^ (h & 7))
        const int pb = g & 1;
        if (g >= 2 && !mbar_wait(&bar->pv_done[pb], ((g >> 1) - 1) & 1, guard)) { ok = false; break; }
        uint8_t* prow = sP + pb * kPBytes + h * 128;
        float lsum = 0.f;
#pragma unroll
        for (int c = 0; c < kNK / 8; ++c) {
          float e[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            e[i] = exp2f(s[c * 8 + i] - m_run);
            lsum += e[i];
          }
          uint4 pk;
          pk.x = pack_bf16x2(e[0], e[1]);
          pk.y = pack_bf16x2(e[2], e[3]);
          pk.z = pack_bf16x2(e[4], e[5]);
          pk.w = pack_bf16x2(e[6], e[7]);
          *reinterpret_cast<uint4*>(prow + ((c ^ (h & 7)) << 4)) = pk;
        }
        l_run += lsum;
        if (nvalid < kNK) {
          // keys past the row's end: zero their latent rows so garbage cannot reach P·V
          uint8_t* st = sKV + (g % kStages) * kStageBytes;
          const int nbytes_row = 128;
          const int chunks = (kNK - nvalid) * (nbytes_row / 16) * 4;
          for (int q = tid; q < chunks; q += 128) {
            const int slab = q / ((kNK - nvalid) * 8);
            const int rem = q - slab * ((kNK - nvalid) * 8);
            const int r = nvalid + rem / 8;
            const int ch = rem & 7;
            *reinterpret_cast<uint4*>(st + slab * kSlabKV + r * 128 + ch * 16) = make_uint4(0, 0, 0, 0);
          }
        }
        fence_async_smem();
        tc_fence_before();
        mbar_arrive(&bar->p_full[pb]);
      }
      if (!ok) break;
      // ------------------------------------------------------------ epilogue of the piece
      const int glast = g - 1;
      if (!mbar_wait(&bar->pv_done[glast & 1], (glast >> 1) & 1, guard)) break;
      tc_fence_after();
      const float inv_l = 1.f / l_run;
      const float lse = (m_run + log2f(l_run)) * 0.69314718055994531f;
      const bool whole = (k0 == 0 && k1 == nrow);
      if (whole) {
        bf16* dst = p.o_lat + (static_cast<size_t>(row) * p.n_heads + h) * kC + col0;
#pragma unroll 1
        for (int c = 0; c < 256 / 16; ++c) {
          float v[16];
          tmem_ld16(tmem + lane_off + kTmemO + c * 16, v);
          if (h < p.n_heads) {
            uint4 a, b;
            a.x = pack_bf16x2(v[0] * inv_l, v[1] * inv_l);
            a.y = pack_bf16x2(v[2] * inv_l, v[3] * inv_l);
            a.z = pack_bf16x2(v[4] * inv_l, v[5] * inv_l);
            a.w = pack_bf16x2(v[6] * inv_l, v[7] * inv_l);
            b.x = pack_bf16x2(v[8] * inv_l, v[9] * inv_l);
            b.y = pack_bf16x2(v[10] * inv_l, v[11] * inv_l);
            b.z = pack_bf16x2(v[12] * inv_l, v[13] * inv_l);
            b.w = pack_bf16x2(v[14] * inv_l, v[15] * inv_l);
            reinterpret_cast<uint4*>(dst + c * 16)[0] = a;
            reinterpret_cast<uint4*>(dst + c * 16)[1] = b;
          }
        }
        if (rank == 0 && p.lse_out && h < p.n_heads)
          p.lse_out[static_cast<size_t>(row) * p.n_heads + h] = lse;
      } else {
        const int slot = first_row ? 0 : 1;
        float* dst = p.part_o + ((static_cast<size_t>(pair) * 2 + slot) * 128 + h) * kC + col0;
#pragma unroll 1
        for (int c = 0; c < 256 / 16; ++c) {
          float v[16];
          tmem_ld16(tmem + lane_off + kTmemO + c * 16, v);
#pragma unroll
          for (int i = 0; i < 16; i += 4)
            *reinterpret_cast<float4*>(dst + c * 16 + i) =
                make_float4(v[i] * inv_l, v[i + 1] * inv_l, v[i + 2] * inv_l, v[i + 3] * inv_l);
        }
        if (rank == 0) p.part_lse[(static_cast<size_t>(pair) * 2 + slot) * 128 + h] = lse;
      }
      tc_fence_before();
      mbar_arrive(&bar->o_empty);
      ++piece;
      it.next();
    }
  }

  // ------------------------------------------------------------------ teardown
  if (warp == 1) {
    int dummy = 0;
    Guard drain{reinterpret_cast<volatile int*>(&dummy), p.status};
    mbar_wait(&bar->drain, 0, drain);   // every MMA this CTA issued has completed
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();   // no remote access into this CTA's shared memory is still pending
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

int attention_pairs() {
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms / 2 > 0 ? sms / 2 : 1;
}

cudaError_t attention_prepare() {
  return cudaFuncSetAttribute(latent_attention_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              kAttnSmem);
}

cudaError_t launch_attention(const CUtensorMap& tq, const CUtensorMap& tkv, const CUtensorMap& tpe,
                             const AttnParams& p, int n_pairs, cudaStream_t s) {
  latent_attention_kernel<<<dim3(2 * n_pairs), dim3(kThreads), kAttnSmem, s>>>(tq, tkv, tpe, p);
  return cudaGetLastError();
}

// ------------------------------------------------------------------------------------------
// Combine: rows cut between pairs merge their normalised partials by log-sum-exp weights.
// ------------------------------------------------------------------------------------------
__device__ __forceinline__ int pair_of_key(long long total, int pairs, long long e) {
  int q = static_cast<int>((e * pairs) / total);
  if (q >= pairs) q = pairs - 1;
  while (q + 1 < pairs && pair_begin(total, pairs, q + 1) <= e) ++q;
  while (q > 0 && pair_begin(total, pairs, q) > e) --q;
  return q;
}

__global__ void __launch_bounds__(256) combine_kernel(const CombineParams p) {
  const int r = blockIdx.x;
  const long long total = p.row_prefix[p.rows];
  const int pairs = active_pairs(total, p.n_pairs, p.min_keys_per_pair);
  const long long R0 = p.row_prefix[r], R1 = p.row_prefix[r + 1];
  const int plo = pair_of_key(total, pairs, R0), phi = pair_of_key(total, pairs, R1 - 1);
  if (plo == phi) return;   // written by one pair
  const int npart = phi - plo + 1;
  for (int h = threadIdx.x >> 5; h < p.n_heads; h += 8) {
    const int lane = threadIdx.x & 31;
    float mx = -INFINITY;
    for (int q = plo; q <= phi; ++q) {
      const int slot = (q == plo && pair_begin(total, pairs, q) < R0) ? 1 : 0;
      mx = fmaxf(mx, p.part_lse[(static_cast<size_t>(q) * 2 + slot) * 128 + h]);
    }
    float wsum = 0.f;
    float acc[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) acc[i] = 0.f;
    for (int q = plo; q <= phi; ++q) {
      const int slot = (q == plo && pair_begin(total, pairs, q) < R0) ? 1 : 0;
      const size_t base = (static_cast<size_t>(q) * 2 + slot) * 128 + h;
      const float w = exp2f((p.part_lse[base] - mx) * 1.4426950408889634f);
      wsum += w;
      const float* src = p.part_o + base * kC;
#pragma unroll
      for (int i = 0; i < 16; ++i) acc[i] += w * src[lane + 32 * i];
    }
    (void)npart;
    const float inv = 1.f / wsum;
    bf16* dst = p.o_lat + (static_cast<size_t>(r) * p.n_heads + h) * kC;
#pragma unroll
    for (int i = 0; i < 16; ++i) dst[lane + 32 * i] = __float2bfloat16_rn(acc[i] * inv);
    if (lane == 0 && p.lse_out)
      p.lse_out[static_cast<size_t>(r) * p.n_heads + h] = mx + logf(wsum);
  }
}

cudaError_t launch_combine(const CombineParams& p, cudaStream_t s) {
  combine_kernel<<<p.rows, 256, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace mla
