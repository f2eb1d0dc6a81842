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
//     (128 rows; heads beyond H are zero rows), so QK^T and P·V are dense 128-row tcgen05 MMAs.
//   * A cluster of TWO CTAs (one SM each) handles a row.  CTA 0 owns the latent columns
//     [0, 256); CTA 1 owns [256, 512) and the 64 rotary columns.  Each CTA streams only its
//     columns of every cache tile (the 576-wide cache row crosses HBM once), computes a partial
//     score tile over them and hands it to the peer; both CTAs then hold identical full scores
//     and run the identical online softmax.  Each CTA accumulates the value half it owns,
//     O[128 x 256] fp32 in TMEM.
//   * The CTA's half of the absorbed query lives in TMEM and is the A operand of the score MMA;
//     the probabilities P (bf16) overwrite the score tile in TMEM and are the A operand of the
//     P·V MMA.  Shared memory holds the cache ring (32-key tiles, 7 stages, TMA with 128-byte
//     swizzle, evict-first) and the exchange buffers.
//     TMEM columns: O [0,256) | query half [256,416) | three 32-column score/P buffers [416,512).
//     With three buffers the score MMA of tile g only waits for P·V of tile g-3, so the tensor
//     core runs two tiles ahead of the softmax.
//   * Score exchange: partial tiles go through a local staging buffer to the bulk-copy engine
//     (shared::cta → the peer's shared memory), which completes a transaction count on the
//     peer's barrier.
//   * Eight softmax warps in two groups of four that take alternate tiles (ping-pong); within a
//     group one thread owns one head row.  Only the running-max decision is handed from tile to
//     tile across the groups (per-row flag in shared memory); each group keeps its own partial
//     row sum, so the softmax work of consecutive tiles overlaps.
//   * Each warp stages its 32 rows of partial scores and ships them with its own 4 KB bulk copy;
//     it waits only for the copy of its counterpart warp (same group and lane quarter) in the
//     peer CTA, through a barrier pair of its own.
//   * The flattened key range of all rows is split evenly over the cluster pairs (split-K over
//     keys, also across row boundaries); a row cut between pairs leaves normalised partials
//     (O/l, lse) for the combine kernel, an uncut row is written as bf16 o_lat directly.
//   * Online softmax in exp2 domain with lazy rescaling: the running max is only raised (and O
//     in TMEM rescaled) when a tile's max exceeds it by more than 8 (factor 256), which keeps the
//     rescale off the common path while the result stays exact.
//   * Warp roles: warp 0 TMA producer, warp 1 TMEM owner + MMA issuer, warps 2-9 query loader,
//     softmax and epilogue (thread pair = head row = TMEM lane).
//   * Every wait is bounded (see tc100.cuh); a stuck pipeline records a status and ends.
#include "internal.h"
#include "tc100.cuh"

namespace mla {

namespace {

constexpr int kNK = kAttnKeysPerTile;      // keys per tile
constexpr int kStages = 7;                 // cache tile ring depth
constexpr int kL2Ahead = 12;               // tiles the L2 prefetch runs ahead of the ring loads
constexpr int kSlabKV = kNK * 128;         // 4 KB: 64 columns x 32 keys, bf16
constexpr int kMaxSlabs = 5;               // rank 1: 4 latent slabs + 1 rotary slab
constexpr int kSlabQ = 128 * 64 * 2;       // 16 KB: 64 query columns of all 128 head rows
constexpr int kStageBytes = kMaxSlabs * kSlabKV;
constexpr int kXSlot = 128 * kNK * 4;      // 16 KB: one partial score tile, fp32

constexpr int kOffKV = 0;
constexpr int kOffX = kOffKV + kStages * kStageBytes;     // receive slots (peer → this CTA)
constexpr int kOffY = kOffX + 2 * kXSlot;                 // staging slots (this CTA → peer)
constexpr int kOffRed = kOffY + 2 * kXSlot;               // row-max / row-sum exchange
constexpr int kOffBar = kOffRed + 3 * 2 * 128 * 4;
constexpr int kAttnSmem = kOffBar + 512 + 1024;

constexpr int kTmemCols = 512;
constexpr uint32_t kTmemO = 0;             // [0, 256)
constexpr uint32_t kTmemQ = 256;           // [256, 416): up to 320 bf16 K-columns
constexpr uint32_t kTmemS = 416;           // three 32-column score / probability buffers
constexpr int kNS = 3;

constexpr int kSoftmaxWarps = 8;
constexpr int kSoftmaxThreads = kSoftmaxWarps * 32;
constexpr int kThreads = 64 + kSoftmaxThreads;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

struct Bars {
  uint64_t kv_full[kStages], kv_empty[kStages];
  uint64_t q_empty;         // the piece's last score MMA has read the query in TMEM
  uint64_t s_full[6], p_full[kNS], pv_done[6];
  uint64_t o_empty;
  uint64_t x_full[8], x_empty[8];   // [group][warp quad]
  uint64_t sync_all;       // the 256 softmax threads
  uint64_t drain;
  uint32_t tmem_slot;
  int abort_flag;
};
static_assert(sizeof(Bars) <= 512, "barrier block");
static_assert(kAttnSmem <= 232448, "shared memory budget");

// Iterates the pieces (row, [k0, k1)) of one pair's key range.
struct PieceIter {
  const long long* prefix;
  int rows;
  long long e0, e1;
  int r;
  // first_row: the row containing key b when known (else -1: binary search)
  __device__ void init(const long long* pf, int nrows, long long b, long long e, int first_row) {
    prefix = pf;
    rows = nrows;
    e0 = b;
    e1 = e;
    r = first_row >= 0 ? first_row : row_of_key(pf, nrows, b);
  }
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

__device__ __forceinline__ uint32_t xbuf_off(int slot, int h, int c) {
  // row h of a slot holds 32 floats = 8 chunks of 16 B; chunk c is stored at (c + h) & 7
  return static_cast<uint32_t>(slot * kXSlot + h * 128 + (((c + h) & 7) << 4));
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    latent_attention_kernel(const __grid_constant__ CUtensorMap tmKV,
                            const __grid_constant__ CUtensorMap tmPE,
                            const __grid_constant__ CUtensorMap tmQ,
                            const __grid_constant__ CUtensorMap tmO,
                            const __grid_constant__ CUtensorMap tmPart, const AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sKV = smem + kOffKV;
  uint8_t* sX = smem + kOffX;
  uint8_t* sY = smem + kOffY;
  float* sRed = reinterpret_cast<float*>(smem + kOffRed);   // m_ref, seq, 2 x row sums
  Bars* bar = reinterpret_cast<Bars*>(smem + kOffBar);

  // Programmatic dependent launch: the key prefix is final before this kernel can start (the
  // RMSNorm kernel publishes it before releasing its dependents) and the cache is an input of the
  // whole chain, so the producer streams cache tiles right away; the warps that read queries or
  // write outputs wait for the previous kernels first.
  pdl_launch_dependents();
  const uint32_t rank = cluster_ctarank();
  const uint32_t peer = rank ^ 1u;
  const int pair = static_cast<int>(cluster_id_x());
  const int launched_pairs = static_cast<int>(nclusters_x());
  const long long total = __ldg(p.row_prefix + p.rows);
  const int row0 = p.pair_row ? __ldg(p.pair_row + pair) : -1;   // same round trip as total
  const int pairs = active_pairs(total, launched_pairs, p.min_keys_per_pair);
  if (pair >= pairs) {         // both CTAs of the pair take this branch together
    pdl_wait();
    return;
  }
  const long long e0 = pair_begin(total, pairs, pair), e1 = pair_begin(total, pairs, pair + 1);

  const int warp = static_cast<int>(warp_id());
  const int nslabs = rank == 0 ? 4 : 5;           // 64-column slabs this CTA owns
  const int col0 = rank == 0 ? 0 : 256;           // first cache / query column it owns
  Guard guard{reinterpret_cast<volatile int*>(&bar->abort_flag), p.status};

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&bar->kv_full[i], 1);
      mbar_init(&bar->kv_empty[i], 1);
    }
    mbar_init(&bar->q_empty, 1);
    for (int i = 0; i < 6; ++i) {
      mbar_init(&bar->s_full[i], 1);
      mbar_init(&bar->pv_done[i], 1);
    }
    for (int i = 0; i < kNS; ++i) mbar_init(&bar->p_full[i], 128);   // the tile's group
    for (int i = 0; i < 8; ++i) {
      mbar_init(&bar->x_full[i], 1);     // receiving warp's expect_tx + the peer warp's 4 KB copy
      mbar_init(&bar->x_empty[i], 1);    // the peer warp has consumed this warp's last copy
    }
    mbar_init(&bar->o_empty, kSoftmaxThreads);
    mbar_init(&bar->sync_all, kSoftmaxThreads);
    mbar_init(&bar->drain, 1);
    bar->abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmKV);
    tma_prefetch_desc(&tmPE);
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmO);
    tma_prefetch_desc(&tmPart);
  }
  if (warp == 1) tmem_alloc(&bar->tmem_slot, kTmemCols);
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();   // the peer's barriers are initialised before any remote arrive
  tc_fence_after();
  const uint32_t tmem = bar->tmem_slot;

  PieceIter it;
  it.init(p.row_prefix, p.rows, e0, e1, row0);

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    // Ring slot sequence per piece: this CTA's query slabs (the 128 x 64 column blocks of the
    // absorbed query it owns, 16 KB each), then the piece's cache tiles.
    if (elect_one()) {
      const uint64_t pol = policy_evict_first();
      // L2 look-ahead: a second cursor over the same tiles, kL2Ahead tiles in front of the ring
      // loads, has the TMA unit pull its tiles into L2, so the bytes in flight from HBM are not
      // limited by the ring's depth.  Its first kL2Ahead tiles go out before the wait below.
      PieceIter pf = it;
      bool pf_live = false, pf_done = false;
      int pf_b = 0, pf_key = 0, pf_end = 0;
      auto prefetch_next = [&]() {
        while (!pf_done) {
          if (pf_live && pf_key < pf_end) {
            for (int i = 0; i < 4; ++i) tma_prefetch_l2_3d(&tmKV, col0 + 64 * i, pf_key, pf_b);
            if (rank == 1) tma_prefetch_l2_3d(&tmPE, 0, pf_key, pf_b);
            pf_key += kNK;
            return;
          }
          if (pf_live) pf.next();
          int r, a, e, n;
          bool fr;
          if (!pf.get(r, a, e, n, fr)) {
            pf_done = true;
            return;
          }
          pf_live = true;
          pf_b = r / p.T;
          pf_key = a;
          pf_end = e;
        }
      };
      for (int i = 0; i < kL2Ahead; ++i) prefetch_next();
      pdl_wait();   // the queries come from the absorption GEMM
      int rs = 0;   // ring slot sequence number
      int last_slot[kStages];
      for (int s = 0; s < kStages; ++s) last_slot[s] = -1;
      int row, k0, k1, nrow;
      bool first_row;
      bool ok = true;
      auto take_slot = [&](uint32_t bytes) -> int {   // next ring slot, armed for `bytes`
        const int s = rs % kStages;
        if (rs >= kStages && !mbar_wait(&bar->kv_empty[s], ((rs / kStages) - 1) & 1, guard))
          return -1;
        mbar_arrive_expect_tx(&bar->kv_full[s], bytes);
        last_slot[s] = rs++;
        return s;
      };
      while (ok && it.get(row, k0, k1, nrow, first_row)) {
        const int b = row / p.T;
        const int ntiles = (k1 - k0 + kNK - 1) / kNK;
        for (int i = 0; i < nslabs && ok; ++i) {
          const int s = take_slot(kSlabQ);
          if (s < 0) { ok = false; break; }
          tma_load_3d(sKV + s * kStageBytes, &tmQ, &bar->kv_full[s], col0 + 64 * i, 0, row);
        }
        for (int j = 0; j < ntiles && ok; ++j) {
          const int s = take_slot(nslabs * kSlabKV);
          if (s < 0) { ok = false; break; }
          uint64_t* fb = &bar->kv_full[s];
          uint8_t* dst = sKV + s * kStageBytes;
          const int key = k0 + j * kNK;
          for (int i = 0; i < 4; ++i)
            tma_load_3d_hint(dst + i * kSlabKV, &tmKV, fb, col0 + 64 * i, key, b, pol);
          if (rank == 1) tma_load_3d_hint(dst + 4 * kSlabKV, &tmPE, fb, 0, key, b, pol);
          prefetch_next();
        }
        it.next();
      }
      if (guard.aborted()) {
        int dummy = 0;
        Guard drain{reinterpret_cast<volatile int*>(&dummy), p.status};
        for (int s = 0; s < kStages; ++s)
          if (last_slot[s] >= 0) mbar_wait(&bar->kv_full[s], (last_slot[s] / kStages) & 1, drain);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (elect_one()) {
      const uint32_t idesc_qk = idesc_bf16(128, kNK, false, false);
      const uint32_t idesc_pv = idesc_bf16(128, 256, false, true);
      int g = 0, pc = 0, rs = 0;
      int row, k0, k1, nrow;
      bool first_row;
      // P·V for tile t (ring slot rt): A = P in TMEM (aliasing the tile's score buffer), B = the
      // stage's four latent slabs, MN-major (64 value columns per slab, keys along K).
      auto issue_pv = [&](int t, int rt, bool first) -> bool {
        const int sb = t % kNS, s = rt % kStages;
        if (!mbar_wait(&bar->p_full[sb], (t / kNS) & 1, guard)) return false;
        if (first && pc > 0 && !mbar_wait(&bar->o_empty, (pc - 1) & 1, guard)) return false;
        tc_fence_after();
        const uint32_t b0 = smem_u32(sKV + s * kStageBytes);
#pragma unroll
        for (int k = 0; k < kNK / 16; ++k) {
          umma_bf16_tmem_a(tmem + kTmemO, tmem + kTmemS + sb * kNK + k * 8,
                           smem_desc_sw128(b0 + k * 2048, kSlabKV, 1024), idesc_pv,
                           (first && k == 0) ? 0u : 1u);
        }
        umma_commit(&bar->kv_empty[s]);
        umma_commit(&bar->pv_done[t % 6]);
        return true;
      };
      bool ok = true;
      while (ok && it.get(row, k0, k1, nrow, first_row)) {
        const int ntiles = (k1 - k0 + kNK - 1) / kNK;
        // the piece's query half → TMEM, once the previous piece's score MMAs have read the old one
        if (pc > 0 && !mbar_wait(&bar->q_empty, (pc - 1) & 1, guard)) break;
        for (int i = 0; i < nslabs && ok; ++i, ++rs) {
          const int s = rs % kStages;
          if (!mbar_wait(&bar->kv_full[s], (rs / kStages) & 1, guard)) { ok = false; break; }
          tc_fence_after();
          const uint32_t q0 = smem_u32(sKV + s * kStageBytes);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            tmem_cp_128x256b(tmem + kTmemQ + i * 32 + kk * 8, smem_desc_sw128(q0 + kk * 32, 16, 1024));
          umma_commit(&bar->kv_empty[s]);
        }
        if (!ok) break;
        const int g0 = g, rs0 = rs;
        for (int j = 0; j < ntiles && ok; ++j, ++g) {
          const int s = (rs0 + j) % kStages, sb = g % kNS;
          if (!mbar_wait(&bar->kv_full[s], ((rs0 + j) / kStages) & 1, guard)) { ok = false; break; }
          tc_fence_after();
          // scores: S[128 x 32] = Q_half (TMEM) x K_half^T (smem, K-major)
          const uint32_t kv0 = smem_u32(sKV + s * kStageBytes);
          for (int i = 0; i < nslabs; ++i) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              umma_bf16_tmem_a(tmem + kTmemS + sb * kNK, tmem + kTmemQ + i * 32 + kk * 8,
                               smem_desc_sw128(kv0 + i * kSlabKV + kk * 32, 16, 1024), idesc_qk,
                               (i | kk) != 0);
            }
          }
          umma_commit(&bar->s_full[g % 6]);
          if (j == ntiles - 1) umma_commit(&bar->q_empty);
          if (j >= 2 && !issue_pv(g - 2, rs0 + j - 2, j - 2 == 0)) { ok = false; break; }
        }
        if (!ok) break;
        // the piece's last (up to two) P·V products
        for (int t = (g - 2 > g0 ? g - 2 : g0); t < g && ok; ++t)
          ok = issue_pv(t, rs0 + (t - g0), t == g0);
        if (!ok) break;
        rs = rs0 + ntiles;
        ++pc;
        it.next();
      }
      umma_commit(&bar->drain);
    }
  } else {
    // ---------------------------------------------------------------- query load, softmax, epilogue
    // Two groups of four warps take alternate tiles (group = global tile index & 1); within a
    // group a thread owns one head row (TMEM lane) and all 32 keys of its tiles.  The running
    // maximum of a row is handed from tile to tile across the groups through m_ref / seq in
    // shared memory; each group keeps its own partial row sum relative to the last maximum it
    // used, so the two groups' softmax work overlaps and only the max decision is sequential.
    const int quad = warp & 3;
    const int grp = (warp - 2) >> 2;                         // 0: warps 2-5, 1: warps 6-9
    const int lane = static_cast<int>(lane_id());
    const int h = quad * 32 + lane;                          // head row = TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const int tid = static_cast<int>(threadIdx.x) - 64;      // 0..255
    const int gtid = tid & 127;                              // thread index within the group
    volatile float* m_ref = reinterpret_cast<volatile float*>(sRed);            // [128]
    volatile int* seq = reinterpret_cast<volatile int*>(sRed + 128);            // [128]
    float* lsum_x = sRed + 256;                                                  // [2][128]
    const uint32_t y_warp = smem_u32(sY) + grp * kXSlot + quad * 4096;         // this warp's rows
    const uint32_t x_warp_remote = mapa_shared(smem_u32(sX), peer) + grp * kXSlot + quad * 4096;
    // exchange barriers are per warp: warp (group, quad) trades its 32 head rows with the peer
    // CTA's warp of the same group and quad only
    const int xw = grp * 4 + quad;
    const uint32_t xfull_remote = mapa_shared(smem_u32(&bar->x_full[xw]), peer);
    const uint32_t xempty_remote = mapa_shared(smem_u32(&bar->x_empty[xw]), peer);
    int g = 0, pc = 0;
    int row, k0, k1, nrow;
    bool first_row;
    bool ok = true;
    uint32_t ph_all = 0;
    auto sync_all = [&]() -> bool {
      mbar_arrive(&bar->sync_all);
      return warp_wait(&bar->sync_all, (ph_all++) & 1, guard);
    };
    pdl_wait();   // outputs may still be read by the kernels before this one
    if (tid < 128) seq[tid] = -1;
    if (!sync_all()) ok = false;

    while (ok && it.get(row, k0, k1, nrow, first_row)) {
      const int ntiles = (k1 - k0 + kNK - 1) / kNK;
      const int g0 = g;
      // ring slot of the piece's first tile: every piece so far (this one included) put its
      // query slabs into the ring ahead of its tiles
      const int rs0 = g0 + nslabs * (pc + 1);

      float l_g = 0.f;              // this group's partial row sum ...
      float m_used = -INFINITY;     // ... relative to this maximum
      int j = ((g0 & 1) == grp) ? 0 : 1;
      for (; j < ntiles; j += 2) {
        const int t = g0 + j;
        const int k = t >> 1;       // per-group tile counter (exchange slot phases)
        // scores of this CTA's columns
        if (!warp_wait(&bar->s_full[t % 6], (t / 6) & 1, guard)) { ok = false; break; }
        tc_fence_after();
        float s[kNK];
        tmem_ld32(tmem + lane_off + kTmemS + (t % kNS) * kNK, s);
        // hand this warp's 32 rows to the peer: stage locally, one bulk copy per warp (measured
        // faster than per-thread st.async stores into the peer's slot)
        if (lane == 0) bulk_wait_read_all();
        __syncwarp();
#pragma unroll
        for (int c = 0; c < kNK / 4; ++c)
          *reinterpret_cast<float4*>(sY + grp * kXSlot + xbuf_off(0, h, c)) =
              make_float4(s[4 * c], s[4 * c + 1], s[4 * c + 2], s[4 * c + 3]);
        fence_async_smem();
        __syncwarp();
        if (lane == 0) {
          if (k >= 1 && !mbar_wait<true>(&bar->x_empty[xw], (k - 1) & 1, guard)) ok = false;
          if (ok) {
            bulk_copy_to_peer(x_warp_remote, y_warp, 4096, xfull_remote);
            bulk_commit();
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        // the peer's half of the same tile
        if (lane == 0) mbar_arrive_expect_tx(&bar->x_full[xw], kXSlot / 4);
        if (!warp_wait<true>(&bar->x_full[xw], k & 1, guard)) { ok = false; break; }
#pragma unroll
        for (int c = 0; c < kNK / 4; ++c) {
          const float4 x =
              *reinterpret_cast<const float4*>(sX + grp * kXSlot + xbuf_off(0, h, c));
          s[4 * c] += x.x;
          s[4 * c + 1] += x.y;
          s[4 * c + 2] += x.z;
          s[4 * c + 3] += x.w;
        }
        // every lane has consumed its loads from the slot before lane 0 lets the peer refill it
        consume32(s);
        __syncwarp();
        if (lane == 0) mbar_arrive_remote_relaxed(xempty_remote);
        const int key0 = k0 + j * kNK;
        const int nvalid = min(kNK, k1 - key0);
        if (p.logits && rank == 0 && h < p.n_heads) {
          float* lg =
              p.logits + (static_cast<size_t>(row) * p.n_heads + h) * p.max_seq_len + key0;
#pragma unroll
          for (int i = 0; i < kNK; ++i)
            if (i < nvalid) lg[i] = s[i] * p.scale;
        }
        // the tile maximum on unscaled scores (the scale is positive: it commutes with max); the
        // exp2 below applies the scale in its FMA
        float mx[8];
        const float c2 = p.scale_log2;
#pragma unroll
        for (int i = 0; i < kNK; ++i) s[i] = i < nvalid ? s[i] : -INFINITY;
#pragma unroll
        for (int i = 0; i < 8; ++i) mx[i] = fmaxf(fmaxf(s[i], s[i + 8]), fmaxf(s[i + 16], s[i + 24]));
#pragma unroll
        for (int i = 0; i < 4; ++i) mx[i] = fmaxf(mx[i], mx[i + 4]);
        const float mt = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * c2;
        // running-max decision for tile t (after the other group decided tile t-1)
        float m_prev = -INFINITY;
        if (j > 0) {
          bool seen = true;
          if (seq[h] != t - 1) {
            const unsigned long long t0 = globaltimer_ns();
            uint32_t n = 0;
            while (seq[h] != t - 1) {
              if ((++n & 63u) == 0 &&
                  (guard.aborted() || globaltimer_ns() - t0 > kWaitLimitNs)) {
                if (!guard.aborted()) guard.fail(kDevTimeout);
                seen = false;
                break;
              }
            }
          }
          if (!__all_sync(0xffffffffu, seen)) { ok = false; break; }
          __threadfence_block();
          m_prev = m_ref[h];
        }
        float m_dec = m_prev;
        const float m_new = fmaxf(m_prev, mt);
        const bool raise = m_new > m_prev + kRescaleThreshold;
        // O holds tiles up to t-1: if any row of the warp raises its maximum, the warp waits for
        // their last P·V and rescales (factor 1 for the other rows) — warp-uniform TMEM access
        if (j > 0 && __any_sync(0xffffffffu, raise)) {
          if (!warp_wait(&bar->pv_done[(t - 1) % 6], ((t - 1) / 6) & 1, guard)) { ok = false; break; }
          tc_fence_after();
          const float f = raise ? fast_exp2(m_prev - m_new) : 1.f;
#pragma unroll 1
          for (int c = 0; c < 256 / 16; ++c) {
            float v[16];
            const uint32_t a = tmem + lane_off + kTmemO + c * 16;
            tmem_ld16(a, v);
#pragma unroll
            for (int i = 0; i < 16; ++i) v[i] *= f;
            tmem_st16(a, v);
          }
          tc_fence_before();
        }
        if (raise) m_dec = m_new;
        m_ref[h] = m_dec;
        __threadfence_block();
        seq[h] = t;
        if (m_used != m_dec) {
          if (m_used != -INFINITY) l_g *= fast_exp2(m_used - m_dec);
          m_used = m_dec;
        }
        // probabilities → TMEM (over the score buffer), row sum
        uint32_t pk[kNK / 2];
        float e[kNK];
#pragma unroll
        for (int i = 0; i < kNK; ++i) e[i] = fast_exp2(fmaf(s[i], c2, -m_dec));
#pragma unroll
        for (int i = 0; i < kNK / 2; ++i) pk[i] = pack_bf16x2(e[2 * i], e[2 * i + 1]);
#pragma unroll
        for (int i = 0; i < 16; ++i) e[i] += e[i + 16];
#pragma unroll
        for (int i = 0; i < 8; ++i) e[i] += e[i + 8];
#pragma unroll
        for (int i = 0; i < 4; ++i) e[i] += e[i + 4];
        l_g += (e[0] + e[2]) + (e[1] + e[3]);
        tmem_st16_u32(tmem + lane_off + kTmemS + (t % kNS) * kNK, pk);
        if (nvalid < kNK) {
          // keys past the piece's end: zero their latent rows so garbage cannot reach P·V
          uint8_t* st = sKV + ((rs0 + j) % kStages) * kStageBytes;
          const int per_slab = (kNK - nvalid) * 8;
          for (int q = gtid; q < per_slab * 4; q += 128) {
            const int slab = q / per_slab;
            const int rem = q - slab * per_slab;
            *reinterpret_cast<uint4*>(st + slab * kSlabKV + (nvalid + (rem >> 3)) * 128 +
                                      ((rem & 7) << 4)) = make_uint4(0, 0, 0, 0);
          }
          fence_async_smem();
        }
        tc_fence_before();
        mbar_arrive(&bar->p_full[t % kNS]);
      }
      if (!ok) break;
      g = g0 + ntiles;

      // ------------------------------------------------------------ epilogue of the piece
      const int glast = g - 1;
      // final maximum of the row (decided at the last tile), both groups' sums relative to it
      {
        bool seen = true;
        const unsigned long long t0 = globaltimer_ns();
        uint32_t n = 0;
        while (seq[h] != glast) {
          if ((++n & 63u) == 0 && (guard.aborted() || globaltimer_ns() - t0 > kWaitLimitNs)) {
            if (!guard.aborted()) guard.fail(kDevTimeout);
            seen = false;
            break;
          }
        }
        if (!__all_sync(0xffffffffu, seen)) break;
      }
      __threadfence_block();
      const float m_fin = m_ref[h];
      lsum_x[grp * 128 + h] = (m_used == -INFINITY) ? 0.f : l_g * fast_exp2(m_used - m_fin);
      if (!sync_all()) break;
      const float l_tot = lsum_x[h] + lsum_x[128 + h];
      if (!warp_wait(&bar->pv_done[glast % 6], (glast / 6) & 1, guard)) break;
      tc_fence_after();
      const float inv_l = 1.f / l_tot;
      const float lse = (m_fin + log2f(l_tot)) * 0.69314718055994531f;
      const bool whole = (k0 == 0 && k1 == nrow);
      const int ocol = col0 + grp * 128;
      const int slot = first_row ? 0 : 1;
      // The warp's 32 rows x 128 columns of O leave through its 4 KB staging slot, one block of
      // 32 rows x 128 bytes at a time (bf16: 64 columns, fp32: 32 columns), written in the
      // 128-byte-swizzle layout (lane = row, 16-byte chunk c at c ^ (row & 7)) and stored by one
      // TMA tile store per block; the warp does not wait for the global writes.
      uint8_t* stg = sY + grp * kXSlot + quad * 4096;
      const int nblk = whole ? 2 : 4;
#pragma unroll 1
      for (int blk = 0; blk < nblk; ++blk) {
        uint32_t w[32];
        if (whole) {
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            float v[32];
            tmem_ld32(tmem + lane_off + kTmemO + grp * 128 + blk * 64 + half * 32, v);
#pragma unroll
            for (int i = 0; i < 16; ++i)
              w[16 * half + i] = pack_bf16x2(v[2 * i] * inv_l, v[2 * i + 1] * inv_l);
          }
        } else {
          float v[32];
          tmem_ld32(tmem + lane_off + kTmemO + grp * 128 + blk * 32, v);
#pragma unroll
          for (int i = 0; i < 32; ++i) w[i] = __float_as_uint(v[i] * inv_l);
        }
        if (blk == nblk - 1) {   // every TMEM read of O is done: the next piece may overwrite it
          tc_fence_before();
          mbar_arrive(&bar->o_empty);
        }
        if (lane == 0) bulk_wait_read_all();   // the slot's last copy or store has read it
        __syncwarp();
#pragma unroll
        for (int c = 0; c < 8; ++c)
          *reinterpret_cast<uint4*>(stg + lane * 128 + ((c ^ (lane & 7)) << 4)) =
              make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
        fence_async_smem();
        __syncwarp();
        if (lane == 0) {
          if (whole) {
            if (quad * 32 < p.n_heads) tma_store_3d(&tmO, stg, ocol + blk * 64, quad * 32, row);
          } else {
            tma_store_2d(&tmPart, stg, ocol + blk * 32, (pair * 2 + slot) * 128 + quad * 32);
          }
          bulk_commit();
        }
      }
      if (whole) {
        if (rank == 0 && grp == 0 && p.lse_out && h < p.n_heads)
          p.lse_out[static_cast<size_t>(row) * p.n_heads + h] = lse;
      } else if (rank == 0 && grp == 0) {
        p.part_lse[(static_cast<size_t>(pair) * 2 + slot) * 128 + h] = lse;
      }
      ++pc;
      it.next();
    }
    if (lane == 0) bulk_wait_all();   // every copy this warp sent has landed in the peer
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

cudaError_t launch_attention(const AttnMaps& m, const AttnParams& p, int n_pairs, cudaStream_t s,
                             bool pdl) {
  LaunchCfg lc(dim3(2 * n_pairs), dim3(kThreads), kAttnSmem, s, pdl);
  return cudaLaunchKernelEx(&lc.cfg, latent_attention_kernel, m.kv, m.pe, m.q, m.o, m.part, p);
}

bool make_attention_maps(AttnMaps* m, const void* kv, int64_t kv_sb, int64_t kv_st, const void* pe,
                         int64_t pe_sb, int64_t pe_st, int batch, int max_seq_len, const void* qabs,
                         int rows, const void* o_lat, int n_heads, const void* part_o, int pairs) {
  const CUtensorMapDataType bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const CUtensorMapSwizzle sw = CU_TENSOR_MAP_SWIZZLE_128B;
  const uint64_t L = static_cast<uint64_t>(max_seq_len), Bt = static_cast<uint64_t>(batch);
  const uint64_t R = static_cast<uint64_t>(rows), H = static_cast<uint64_t>(n_heads);
  const uint32_t box_kv[3] = {64, static_cast<uint32_t>(kNK), 1};
  const uint64_t d_kv[3] = {kC, L, Bt}, s_kv[2] = {static_cast<uint64_t>(kv_st) * 2,
                                                   static_cast<uint64_t>(kv_sb) * 2};
  const uint64_t d_pe[3] = {kDr, L, Bt}, s_pe[2] = {static_cast<uint64_t>(pe_st) * 2,
                                                    static_cast<uint64_t>(pe_sb) * 2};
  const uint64_t d_q[3] = {kDk, kHPad, R}, s_q[2] = {kDk * 2, kHPad * kDk * 2};
  const uint32_t box_q[3] = {64, 128, 1};
  const uint64_t d_o[3] = {kC, H, R}, s_o[2] = {kC * 2, H * kC * 2};
  const uint32_t box_o[3] = {64, 32, 1};
  const uint64_t d_p[2] = {kC, static_cast<uint64_t>(pairs) * 2 * 128}, s_p[1] = {kC * 4};
  const uint32_t box_p[2] = {32, 32};
  return encode_tiled(&m->kv, bf, 3, kv, d_kv, s_kv, box_kv, sw) &&
         encode_tiled(&m->pe, bf, 3, pe, d_pe, s_pe, box_kv, sw) &&
         encode_tiled(&m->q, bf, 3, qabs, d_q, s_q, box_q, sw) &&
         encode_tiled(&m->o, bf, 3, o_lat, d_o, s_o, box_o, sw) &&
         encode_tiled(&m->part, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, part_o, d_p, s_p, box_p, sw);
}

// ------------------------------------------------------------------------------------------
// Combine: rows cut between pairs merge their normalised partials by log-sum-exp weights.
// One warp per (row, head) task; lane l owns columns l, l+32, ..., l+480.
// ------------------------------------------------------------------------------------------
__device__ __forceinline__ int pair_of_key(long long total, int pairs, long long e) {
  int q = static_cast<int>((e * pairs) / total);
  if (q >= pairs) q = pairs - 1;
  while (q + 1 < pairs && pair_begin(total, pairs, q + 1) <= e) ++q;
  while (q > 0 && pair_begin(total, pairs, q) > e) --q;
  return q;
}

// Persistent grid (one block per SM, launched once): each warp walks (row, head) tasks.
constexpr int kCombineThreads = 512;

__global__ void __launch_bounds__(kCombineThreads) combine_kernel(const CombineParams p) {
  pdl_launch_dependents();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int warps = gridDim.x * (kCombineThreads / 32);
  const long long total = p.row_prefix[p.rows];
  const int pairs = active_pairs(total, p.n_pairs, p.min_keys_per_pair);
  for (int task = blockIdx.x * (kCombineThreads / 32) + (threadIdx.x >> 5);
       task < p.rows * p.n_heads; task += warps) {
  const int r = task / p.n_heads, h = task - r * p.n_heads;
  const long long R0 = p.row_prefix[r], R1 = p.row_prefix[r + 1];
  const int plo = pair_of_key(total, pairs, R0), phi = pair_of_key(total, pairs, R1 - 1);
  if (plo == phi) continue;   // written by one pair
  // online log-sum-exp merge, four pieces' loads in flight at a time
  constexpr int kBatch = 4;
  float mx = -INFINITY, wsum = 0.f;
  float acc[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) acc[i] = 0.f;
  for (int q0 = plo; q0 <= phi; q0 += kBatch) {
    float lse[kBatch], v[kBatch][16];
#pragma unroll
    for (int b = 0; b < kBatch; ++b) {
      const int q = q0 + b;
      lse[b] = -INFINITY;
      if (q <= phi) {
        const int slot = (q == plo && pair_begin(total, pairs, q) < R0) ? 1 : 0;
        const size_t base = (static_cast<size_t>(q) * 2 + slot) * 128 + h;
        lse[b] = __ldg(p.part_lse + base);
        const float* src = p.part_o + base * kC;
#pragma unroll
        for (int i = 0; i < 16; ++i) v[b][i] = __ldg(src + lane + 32 * i);
      }
    }
    float m_new = mx;
#pragma unroll
    for (int b = 0; b < kBatch; ++b) m_new = fmaxf(m_new, lse[b]);
    const float f = mx == -INFINITY ? 0.f : exp2f((mx - m_new) * 1.4426950408889634f);
    wsum *= f;
#pragma unroll
    for (int i = 0; i < 16; ++i) acc[i] *= f;
#pragma unroll
    for (int b = 0; b < kBatch; ++b) {
      if (q0 + b <= phi) {
        const float w = exp2f((lse[b] - m_new) * 1.4426950408889634f);
        wsum += w;
#pragma unroll
        for (int i = 0; i < 16; ++i) acc[i] = fmaf(w, v[b][i], acc[i]);
      }
    }
    mx = m_new;
  }
  const float inv = 1.f / wsum;
  bf16* dst = p.o_lat + (static_cast<size_t>(r) * p.n_heads + h) * kC;
#pragma unroll
  for (int i = 0; i < 16; ++i) dst[lane + 32 * i] = __float2bfloat16_rn(acc[i] * inv);
  if (lane == 0 && p.lse_out) p.lse_out[static_cast<size_t>(r) * p.n_heads + h] = mx + logf(wsum);
  }
}

cudaError_t launch_combine(const CombineParams& p, cudaStream_t s, bool pdl) {
  const long long tasks = static_cast<long long>(p.rows) * p.n_heads;
  const long long want = (tasks + kCombineThreads / 32 - 1) / (kCombineThreads / 32);
  const int cap = 2 * attention_pairs();   // one block per SM (registers allow one)
  LaunchCfg lc(dim3(static_cast<unsigned>(want < cap ? want : cap)), dim3(kCombineThreads), 0, s,
               pdl);
  return cudaLaunchKernelEx(&lc.cfg, combine_kernel, p);
}

}  // namespace mla
