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
//     [0, 256) and rotary columns [0, 32); CTA 1 owns [256, 512) and rotary [32, 64), so both
//     move 18 KB per 32-key tile (with all 64 rotary columns on CTA 1 it moved 20 KB against 16
//     and set the pace).  Each CTA streams only its
//     columns of every cache tile (the 576-wide cache row crosses HBM once), computes a partial
//     score tile over them and hands it to the peer; both CTAs then hold identical full scores
//     and run the identical online softmax.  Each CTA accumulates the value half it owns,
//     O[128 x 256] fp32 in TMEM.
//   * The CTA's 256 latent query columns live in TMEM (A operand of the score MMA); its 32
//     rotary query columns stay in shared memory (A from a smem descriptor for those K-steps), so
//     both CTAs have room for four score buffers.  The query reaches TMEM by TMA into ring slots
//     and tcgen05.cp, once per piece.  The probabilities P (bf16) overwrite the score tile in
//     TMEM and are the A operand of P·V.  Shared memory holds the cache ring (32-key tiles, 8
//     stages; latent slabs with 128-byte swizzle, rotary half slabs with 64-byte swizzle;
//     evict-first) and the exchange buffers.
//     TMEM columns: O [0,256) | latent query [256,384) | four 32-column score/P buffers [384,512).
//     With four buffers the score MMA of tile g only waits for P·V of tile g-4 to be issued.
//   * Score exchange: each warp stages its 32 rows of partial scores and ships them with one
//     4 KB bulk copy (shared::cta → the peer's receive slot), which completes a transaction count
//     on the peer warp's own barrier; a warp waits only for its counterpart (same group and lane
//     quarter) in the peer CTA.  The four warps of a lane quarter share one staging slot, handed
//     from use to use in a fixed order.
//   * Twelve softmax warps in three groups of four take turns by tile; within a group one thread
//     owns one head row.  Only the running-max decision is handed from tile to tile across the
//     groups (per-row flag in shared memory); each group keeps its own partial row sum, so the
//     softmax work of consecutive tiles overlaps.
//   * The flattened key range of all rows is split evenly over the cluster pairs (split-K over
//     keys, also across row boundaries); a row cut between pairs leaves normalised partials
//     (O/l, lse) for the combine kernel, an uncut row is written as bf16 o_lat directly, both
//     by TMA tile stores from a swizzled staging block.
//   * Online softmax in exp2 domain with lazy rescaling: the running max is only raised (and O
//     in TMEM rescaled) when a tile's max exceeds it by more than 8 (factor 256), which keeps the
//     rescale off the common path while the result stays exact.
//   * Warp roles: warp 0 TMA producer (lane 1: the CTA's rotary query columns; in the index-mask
//     mode lanes 0-7 gather the cache rows by index and lane 31 loads the rotary query), warp 1 TMEM owner
//     + score-MMA issuer (and the query copies), warp 2 P·V issuer, warps 3-14 softmax and
//     epilogue (thread = head row = TMEM lane).  A tcgen05 instruction costs a single issuing
//     thread ~48 cycles, so the score and P·V streams are issued by two threads in parallel.
//     The score buffer a QK reuses is handed back by the P·V thread's completion barrier.
//   * Every wait is bounded (see tc100.cuh); a stuck pipeline records a status and ends.
#include "internal.h"
#include "tc100.cuh"

namespace mla {

namespace {

constexpr int kNK = kAttnKeysPerTile;      // keys per tile
constexpr int kStages = 8;                 // cache tile ring depth
// L2 look-ahead (build-time tuning): tiles it runs ahead of the ring loads, and one tile in
// kL2Every is prefetched (0: no look-ahead)
#ifndef MLA_ATTN_L2_AHEAD
#define MLA_ATTN_L2_AHEAD 12
#endif
#ifndef MLA_ATTN_L2_EVERY
#define MLA_ATTN_L2_EVERY 3
#endif
constexpr int kL2Ahead = MLA_ATTN_L2_AHEAD;
constexpr int kL2Every = MLA_ATTN_L2_EVERY;
constexpr int kSlabKV = kNK * 128;         // 4 KB: 64 latent columns x 32 keys, bf16
constexpr int kSlabPe = kNK * 64;          // 2 KB: 32 rotary columns x 32 keys (64-byte rows)
constexpr int kSlabQ = 128 * 64 * 2;       // 16 KB: 64 query columns of all 128 head rows
constexpr int kSlabQPe = 128 * 32 * 2;     // 8 KB: this CTA's 32 rotary query columns
constexpr int kTileBytes = 4 * kSlabKV + kSlabPe;   // 18 KB: a CTA's share of a 32-key tile
constexpr int kStageBytes = kTileBytes;    // a ring slot: a tile share or a 16 KB query slab
constexpr int kGroups = 3;                 // softmax groups (4 warps each) taking turns by tile
constexpr int kXWarp = 32 * kNK * 4;       // 4 KB: one warp's 32 rows of a partial score tile

constexpr int kOffKV = 0;
constexpr int kOffX = kOffKV + kStages * kStageBytes;     // receive slots (peer → this CTA), per warp
constexpr int kOffY = kOffX + kGroups * 4 * kXWarp;       // staging slots, one per lane quarter
constexpr int kOffQPe = kOffY + 4 * kXWarp;               // this CTA's rotary query columns
constexpr int kOffRed = kOffQPe + kSlabQPe;               // row-max / row-sum exchange
constexpr int kOffBar = kOffRed + (2 + 2 * kGroups) * 128 * 4;
constexpr int kAttnSmem = kOffBar + 768 + 1024;

constexpr int kTmemCols = 512;
constexpr uint32_t kTmemO = 0;             // [0, 256)
constexpr uint32_t kTmemQ = 256;           // [256, 384): 256 bf16 latent query columns
constexpr uint32_t kTmemS = 384;           // four 32-column score / probability buffers
constexpr int kNS = 4;
constexpr int kNB = 8;                     // ring of per-tile barrier slots (s_full, pv_done)

constexpr int kSoftmaxWarps = 4 * kGroups;
constexpr int kSoftmaxThreads = kSoftmaxWarps * 32;
constexpr int kThreads = 96 + kSoftmaxThreads;
constexpr int kSoftmaxWarp0 = 3;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

struct Bars {
  uint64_t kv_full[kStages], kv_empty[kStages];
  uint64_t q_empty;         // the piece's last score MMA has read the query (TMEM and smem)
  uint64_t qpe_full;        // the piece's rotary query columns (this CTA's 32) have landed
  uint64_t s_full[kNB], p_full[kNS], pv_done[kNB];
  uint64_t o_empty;
  uint64_t x_full[4 * kGroups], x_empty[4 * kGroups];   // [group][warp quad]
  uint64_t sync_all;        // all softmax threads
  uint64_t drain;
  uint32_t tmem_slot;
  int abort_flag;
  // staging slot of each lane quarter: number of uses that have released it (a counter, not a
  // barrier: a warp may start waiting for its turn more than one use ahead)
  int y_released[4];
};
static_assert(sizeof(Bars) <= 768, "barrier block");
static_assert(kAttnSmem <= 232448, "shared memory budget");

// Iterates the pieces (row, [k0, k1)) of one pair's key range.
struct PieceIter {
  const long long* prefix;
  int rows;
  long long e0, e1;
  long long max_keys;   // keys a row can have (cache rows per sequence)
  int r;
  // first_row: the row containing key b when known (else -1: binary search)
  __device__ void init(const long long* pf, int nrows, long long b, long long e, int first_row,
                       long long maxk) {
    prefix = pf;
    rows = nrows;
    e0 = b;
    e1 = e;
    max_keys = maxk;
    r = first_row >= 0 && first_row < nrows ? first_row : row_of_key(pf, nrows, b);
  }
  // Key counts come from the key prefix (written by the RMSNorm kernel of the same call) and are
  // read at L2 (coherent) so every role of the CTA pair sees the same pieces; a record that
  // cannot come from a valid prefix ends the walk (and is reported by the caller's check).
  __device__ bool get(int& row, int& k0, int& k1, int& nkeys_row, bool& first_row) const {
    if (r < 0 || r >= rows) return false;
    const long long R0 = __ldcg(prefix + r), R1 = __ldcg(prefix + r + 1);
    if (R0 >= e1 || R0 < 0 || R1 < R0 || R1 - R0 > max_keys) return false;
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
    latent_attention_kernel(const __grid_constant__ CUtensorMap tmKV,
                            const __grid_constant__ CUtensorMap tmPE,
                            const __grid_constant__ CUtensorMap tmQ,
                            const __grid_constant__ CUtensorMap tmQPe,
                            const __grid_constant__ CUtensorMap tmO,
                            const __grid_constant__ CUtensorMap tmPart,
                            const __grid_constant__ CUtensorMap tmKV2,
                            const __grid_constant__ CUtensorMap tmPE2, const AttnParams p) {
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
  const long long total = __ldcg(p.row_prefix + p.rows);
  const int row0 = p.pair_row ? __ldcg(p.pair_row + pair) : -1;   // same round trip as total
  const int pairs = active_pairs(total, launched_pairs, p.min_keys_per_pair);
  if (pair >= pairs) {         // both CTAs of the pair take this branch together
    pdl_wait();
    return;
  }
  const long long e0 = pair_begin(total, pairs, pair), e1 = pair_begin(total, pairs, pair + 1);

  const int warp = static_cast<int>(warp_id());
  const int col0 = rank == 0 ? 0 : 256;           // first latent cache / query column it owns
  const int pe0 = rank == 0 ? 0 : 32;             // first rotary column it owns
  uint8_t* sQPe = smem + kOffQPe;                 // this CTA's rotary query columns
  Guard guard{reinterpret_cast<volatile int*>(&bar->abort_flag), p.status,
              p.wait_limit_ns ? p.wait_limit_ns : kWaitLimitNs};

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&bar->kv_full[i], 1);
      mbar_init(&bar->kv_empty[i], 1);
    }
    mbar_init(&bar->q_empty, 1);
    mbar_init(&bar->qpe_full, 1);
    for (int i = 0; i < kNB; ++i) {
      mbar_init(&bar->s_full[i], 1);
      mbar_init(&bar->pv_done[i], 1);
    }
    for (int i = 0; i < kNS; ++i) mbar_init(&bar->p_full[i], 128);   // the tile's group
    for (int i = 0; i < 4 * kGroups; ++i) {
      mbar_init(&bar->x_full[i], 1);     // receiving warp's expect_tx + the peer warp's 4 KB copy
      mbar_init(&bar->x_empty[i], 1);    // the peer warp has consumed this warp's last copy
    }
    for (int i = 0; i < 4; ++i) bar->y_released[i] = 0;
    mbar_init(&bar->o_empty, kSoftmaxThreads);
    mbar_init(&bar->sync_all, kSoftmaxThreads);
    mbar_init(&bar->drain, 2);   // both MMA-issuing threads
    bar->abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmKV);
    tma_prefetch_desc(&tmPE);
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmQPe);
    tma_prefetch_desc(&tmO);
    tma_prefetch_desc(&tmPart);
    if (p.topk_idx) {
      tma_prefetch_desc(&tmKV2);
      tma_prefetch_desc(&tmPE2);
    }
  }
  if (warp == 1) tmem_alloc(&bar->tmem_slot, kTmemCols);
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();   // the peer's barriers are initialised before any remote arrive
  tc_fence_after();
  const uint32_t tmem = bar->tmem_slot;

  PieceIter it;
  it.init(p.row_prefix, p.rows, e0, e1, row0, p.max_seq_len);
  // The ring slot each stage was last armed for, and the rotary query slabs armed, by the thread
  // that armed them: if any role gives up, these loads land before the CTA releases its memory.
  int last_slot[kStages];
  for (int s = 0; s < kStages; ++s) last_slot[s] = -1;
  int qpe_armed = 0;

  // lane of warp 0 that loads the CTA's rotary query columns (lanes 0-7 gather in the index-mask
  // mode)
  const uint32_t qpe_lane = p.topk_idx ? 31u : 1u;
  if (warp == 0 && p.topk_idx && lane_id() < 8) {
    // ---------------------------------------------------------------- TMA producer, index mask
    // Key j of a row is cache row topk_idx[row][j] of its sequence: every tile's 32 rows are
    // gathered four at a time (tile::gather4 on the 2-D row maps, one-row boxes), lane l taking
    // keys 4l .. 4l+3 of each slab.  Slots past the piece's end load the piece's first key (a
    // valid row; its score is masked and its latent row zeroed before P·V).  Lane 0 also loads
    // the query slabs and owns the ring bookkeeping.
    const int lane = static_cast<int>(lane_id());
    const uint64_t pol = policy_evict_first();
    pdl_wait();
    int rs = 0;
    int row, k0, k1, nrow;
    bool first_row;
    bool ok = true, bad = false;
    auto take_slot = [&](uint32_t bytes) -> int {   // lane 0: next ring slot, armed for `bytes`
      const int s = rs % kStages;
      if (rs >= kStages && !mbar_wait(&bar->kv_empty[s], ((rs / kStages) - 1) & 1, guard))
        return -1;
      mbar_arrive_expect_tx(&bar->kv_full[s], bytes);
      last_slot[s] = rs++;
      return s;
    };
    while (ok && it.get(row, k0, k1, nrow, first_row)) {
      const long long rowbase = static_cast<long long>(row / p.T) * p.seq_rows;
      const int32_t* idx = p.topk_idx + static_cast<size_t>(row) * p.topk_k;
      const int ntiles = (k1 - k0 + kNK - 1) / kNK;
      if (lane == 0) {
        for (int i = 0; i < 4 && ok; ++i) {
          const int s = take_slot(kSlabQ);
          if (s < 0) { ok = false; break; }
          tma_load_3d(sKV + s * kStageBytes, &tmQ, &bar->kv_full[s], col0 + 64 * i, 0, row);
        }
      }
      ok = __shfl_sync(0xffu, ok, 0);
      int first = __ldg(idx + k0);
      if (first < 0 || first >= p.seq_rows) {
        bad = true;
        first = 0;
      }
      for (int j = 0; j < ntiles && ok; ++j) {
        int rr[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int key = k0 + j * kNK + 4 * lane + i;
          int t = first;
          if (key < k1) {
            t = __ldg(idx + key);
            if (t < 0 || t >= p.seq_rows) {
              bad = true;
              t = 0;
            }
          }
          rr[i] = static_cast<int>(rowbase + t);
        }
        int s = 0;
        if (lane == 0) s = take_slot(kTileBytes);
        s = __shfl_sync(0xffu, s, 0);
        if (s < 0) { ok = false; break; }
        uint64_t* fb = &bar->kv_full[s];
        uint8_t* dst = sKV + s * kStageBytes;
        for (int i = 0; i < 4; ++i)
          tma_gather4(dst + i * kSlabKV + lane * 512, &tmKV2, fb, col0 + 64 * i, rr[0], rr[1],
                      rr[2], rr[3], pol);
        tma_gather4(dst + 4 * kSlabKV + lane * 256, &tmPE2, fb, pe0, rr[0], rr[1], rr[2], rr[3],
                    pol);
      }
      it.next();
    }
    if (bad) atomicCAS(p.status, kDevOk, kDevBadArg);
  } else if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    // Lane 0: ring slot sequence per piece = the 4 latent query slabs this CTA owns (128 x 64
    // columns, 16 KB each), then the piece's cache tiles.  Lane qpe_lane: the piece's 32 rotary
    // query columns of this CTA into their own buffer, once the previous piece's last score MMA
    // has read them.
    const uint32_t lane = lane_id();
    if (lane == 0 && !p.topk_idx) {
      // decode reads each cache row once (evict first); a prefill chunk's rows all re-read the
      // same key prefix, which should stay in L2 (evict last, and no look-ahead: after the first
      // row's pass every tile is an L2 hit)
      const bool reread = p.T > 1;
      const uint64_t pol = reread ? policy_evict_last() : policy_evict_first();
      // L2 look-ahead: a second cursor over the same tiles, kL2Ahead tiles in front of the ring
      // loads, has the TMA unit pull its tiles into L2, so the bytes in flight from HBM are not
      // limited by the ring's depth.  Its first kL2Ahead tiles go out before the wait below.
      // Only one tile in three is prefetched: the prefetches go through the same TMA unit as the
      // ring's loads (~48 GB/s per SM), so prefetching every tile halves the rate at which the
      // ring can be filled; the tiles in between load from HBM within the ring's depth (every
      // tile: 0.83 us per tile; every other: 68.5 us per launch; one in three: 67.0 us).
      PieceIter pf = it;
      bool pf_live = false, pf_done = reread;
      int pf_b = 0, pf_key = 0, pf_end = 0, pf_n = 0;
      auto prefetch_next = [&]() {
        while (!pf_done) {
          if (pf_live && pf_key < pf_end) {
            if (kL2Every > 0 && (pf_n++ % (kL2Every > 0 ? kL2Every : 1)) == 0) {
              for (int i = 0; i < 4; ++i) tma_prefetch_l2_3d(&tmKV, col0 + 64 * i, pf_key, pf_b);
              tma_prefetch_l2_3d(&tmPE, pe0, pf_key, pf_b);
            }
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
        for (int i = 0; i < 4 && ok; ++i) {
          const int s = take_slot(kSlabQ);
          if (s < 0) { ok = false; break; }
          tma_load_3d(sKV + s * kStageBytes, &tmQ, &bar->kv_full[s], col0 + 64 * i, 0, row);
        }
        for (int j = 0; j < ntiles && ok; ++j) {
          const int s = take_slot(kTileBytes);
          if (s < 0) { ok = false; break; }
          uint64_t* fb = &bar->kv_full[s];
          uint8_t* dst = sKV + s * kStageBytes;
          const int key = k0 + j * kNK;
          for (int i = 0; i < 4; ++i)
            tma_load_3d_hint(dst + i * kSlabKV, &tmKV, fb, col0 + 64 * i, key, b, pol);
          tma_load_3d_hint(dst + 4 * kSlabKV, &tmPE, fb, pe0, key, b, pol);
          prefetch_next();
        }
        it.next();
      }
    } else if (lane == qpe_lane) {
      pdl_wait();
      int row, k0, k1, nrow, pc = 0;
      bool first_row;
      while (it.get(row, k0, k1, nrow, first_row)) {
        if (pc > 0 && !mbar_wait(&bar->q_empty, (pc - 1) & 1, guard)) break;
        mbar_arrive_expect_tx(&bar->qpe_full, kSlabQPe);
        tma_load_3d(sQPe, &tmQPe, &bar->qpe_full, kC + pe0, 0, row);
        qpe_armed = ++pc;
        it.next();
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- score-MMA issuer
    if (elect_one()) {
      const uint32_t idesc_qk = idesc_bf16(128, kNK, false, false);
      int g = 0, pc = 0, rs = 0;
      int row, k0, k1, nrow;
      bool first_row;
      const uint32_t qpe0 = smem_u32(sQPe);
      bool ok = true;
      while (ok && it.get(row, k0, k1, nrow, first_row)) {
        const int ntiles = (k1 - k0 + kNK - 1) / kNK;
        // the piece's latent query half → TMEM, once the previous piece's score MMAs have read the
        // old one (its rotary slab is reloaded by the producer after the same point)
        if (pc > 0 && !mbar_wait(&bar->q_empty, (pc - 1) & 1, guard)) break;
        for (int i = 0; i < 4 && ok; ++i, ++rs) {
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
        if (!mbar_wait(&bar->qpe_full, pc & 1, guard)) break;
        const int rs0 = rs;
        for (int j = 0; j < ntiles && ok; ++j, ++g) {
          const int s = (rs0 + j) % kStages, sb = g % kNS;
          if (!mbar_wait(&bar->kv_full[s], ((rs0 + j) / kStages) & 1, guard)) { ok = false; break; }
          // the score buffer held P of tile g - kNS: its P·V (other thread) must have completed
          if (g >= kNS && !mbar_wait(&bar->pv_done[(g - kNS) % kNB], ((g - kNS) / kNB) & 1, guard)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // scores: S[128 x 32] = Q_part x K_part^T over this CTA's 256 latent and 32 rotary
          // columns: latent part with the query in TMEM, rotary part with the query in shared
          // memory (64-byte-swizzled 32-column slabs); cache K-major in smem
          const uint32_t kv0 = smem_u32(sKV + s * kStageBytes);
          for (int i = 0; i < 4; ++i) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              umma_bf16_tmem_a(tmem + kTmemS + sb * kNK, tmem + kTmemQ + i * 32 + kk * 8,
                               smem_desc_sw128(kv0 + i * kSlabKV + kk * 32, 16, 1024), idesc_qk,
                               (i | kk) != 0);
            }
          }
#pragma unroll
          for (int kk = 0; kk < 2; ++kk) {
            umma_bf16(tmem + kTmemS + sb * kNK, smem_desc_sw64(qpe0 + kk * 32, 512),
                      smem_desc_sw64(kv0 + 4 * kSlabKV + kk * 32, 512), idesc_qk, 1u);
          }
          umma_commit(&bar->s_full[g % kNB]);
          if (j == ntiles - 1) umma_commit(&bar->q_empty);
        }
        if (!ok) break;
        rs = rs0 + ntiles;
        ++pc;
        it.next();
      }
      umma_commit(&bar->drain);
    }
  } else if (warp == 2) {
    // ---------------------------------------------------------------- P·V issuer
    // P·V for tile t: A = P in TMEM (aliasing the tile's score buffer), B = the ring stage's four
    // latent slabs, MN-major (64 value columns per slab, keys along K).  P is complete (p_full)
    // only after the score MMA of the tile has finished reading the stage.
    if (elect_one()) {
      const uint32_t idesc_pv = idesc_bf16(128, 256, false, true);
      int g = 0, pc = 0;
      int row, k0, k1, nrow;
      bool first_row;
      bool ok = true;
      while (ok && it.get(row, k0, k1, nrow, first_row)) {
        const int ntiles = (k1 - k0 + kNK - 1) / kNK;
        const int rs0 = g + 4 * (pc + 1);   // ring slot of the piece's first tile
        for (int j = 0; j < ntiles && ok; ++j, ++g) {
          const int sb = g % kNS, s = (rs0 + j) % kStages;
          if (!mbar_wait(&bar->p_full[sb], (g / kNS) & 1, guard)) { ok = false; break; }
          if (j == 0 && pc > 0 && !mbar_wait(&bar->o_empty, (pc - 1) & 1, guard)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t b0 = smem_u32(sKV + s * kStageBytes);
#pragma unroll
          for (int k = 0; k < kNK / 16; ++k) {
            umma_bf16_tmem_a(tmem + kTmemO, tmem + kTmemS + sb * kNK + k * 8,
                             smem_desc_sw128(b0 + k * 2048, kSlabKV, 1024), idesc_pv,
                             (j == 0 && k == 0) ? 0u : 1u);
          }
          umma_commit(&bar->kv_empty[s]);
          umma_commit(&bar->pv_done[g % kNB]);
        }
        if (!ok) break;
        ++pc;
        it.next();
      }
      umma_commit(&bar->drain);
    }
  } else {
    // ---------------------------------------------------------------- softmax, epilogue
    // kGroups groups of four warps take turns by tile (group = global tile index % kGroups);
    // within a group a thread owns one head row (TMEM lane) and all 32 keys of its tiles.  The
    // running maximum of a row is handed from tile to tile across the groups through m_ref / seq
    // in shared memory; each group keeps its own partial row sum relative to the last maximum it
    // used, so the groups' softmax work overlaps and only the max decision is sequential.
    //
    // Staging: the four warps of a lane quarter (one per group) share one 4 KB slot for their
    // outgoing score copies and for the epilogue's TMA stores.  Uses of a slot are numbered in a
    // fixed order (the pieces' tiles, then each piece's epilogue blocks, group 0 before group 1)
    // and handed on through a release counter: use u waits until u uses have released it.
    const int quad = warp & 3;
    const int grp = (warp - kSoftmaxWarp0) >> 2;             // warps 3-6, 7-10, 11-14
    const int lane = static_cast<int>(lane_id());
    const int h = quad * 32 + lane;                          // head row = TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const int tid = static_cast<int>(threadIdx.x) - 32 * kSoftmaxWarp0;   // 0..kSoftmaxThreads-1
    const int gtid = tid & 127;                              // thread index within the group
    volatile float* m_ref = reinterpret_cast<volatile float*>(sRed);            // [128]
    volatile int* seq = reinterpret_cast<volatile int*>(sRed + 128);            // [128]
    float* lsum_x = sRed + 256;                       // [piece parity][kGroups][128]
    uint8_t* stg = sY + quad * kXWarp;                       // this lane quarter's staging slot
    const int xw = grp * 4 + quad;                           // this warp's receive slot / barriers
    uint8_t* xslot = sX + xw * kXWarp;
    const uint32_t x_remote = mapa_shared(smem_u32(xslot), peer);
    const uint32_t xfull_remote = mapa_shared(smem_u32(&bar->x_full[xw]), peer);
    const uint32_t xempty_remote = mapa_shared(smem_u32(&bar->x_empty[xw]), peer);
    // row r of a warp's 4 KB score block: 32 floats = 8 chunks of 16 B, chunk c at (c + r) & 7
    auto xoff = [](int r, int c) -> int { return r * 128 + (((c + r) & 7) << 4); };
    volatile int* y_released = bar->y_released + quad;
    auto acquire_stage = [&](int u) -> bool {   // wait until uses 0..u-1 released the slot
      bool got = true;
      if (*y_released < u) {
        const unsigned long long t0 = globaltimer_ns();
        uint32_t n = 0;
        while (*y_released < u) {
          if ((++n & 63u) == 0 && (guard.aborted() || globaltimer_ns() - t0 > guard.limit_ns)) {
            if (!guard.aborted()) guard.fail(kDevTimeout);
            got = false;
            break;
          }
        }
      }
      got = __all_sync(0xffffffffu, got);
      __threadfence_block();
      return got;
    };
    auto release_stage = [&](int u) {           // the slot's copy / store has read it: hand on
      if (lane == 0) {
        bulk_wait_read_all();
        __threadfence_block();
        *y_released = u + 1;
      }
    };
    int g = 0, pc = 0, ubase = 0;   // tiles before this piece, pieces, extra slot uses before
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
      // four query slabs into the ring ahead of its tiles
      const int rs0 = g0 + 4 * (pc + 1);
      const bool whole = (k0 == 0 && k1 == nrow);
      constexpr int nblk = 2;           // epilogue blocks of 64 columns per writing group
      // group 1 stages its epilogue in its own receive slot when it had a tile in this piece (the
      // peer may refill that slot only after the epilogue: its last release is held back);
      // otherwise it queues on the lane quarter's shared slot behind group 0
      const bool g1_has_tile = ((1 - g0 % kGroups + kGroups) % kGroups) < ntiles;
      bool xe_held = false;

      float l_g = 0.f;              // this group's partial row sum ...
      float m_used = -INFINITY;     // ... relative to this maximum
      int j = ((grp - g0 % kGroups) + kGroups) % kGroups;
      for (; j < ntiles; j += kGroups) {
        const int t = g0 + j;
        const int k = t / kGroups;  // per-group tile counter (exchange slot phases)
        // scores of this CTA's columns
        if (!warp_wait(&bar->s_full[t % kNB], (t / kNB) & 1, guard)) { ok = false; break; }
        tc_fence_after();
        float s[kNK];
        tmem_ld32(tmem + lane_off + kTmemS + (t % kNS) * kNK, s);
        // hand this warp's 32 rows to the peer: stage locally, one 4 KB bulk copy per warp
        if (!acquire_stage(t + ubase)) { ok = false; break; }
#pragma unroll
        for (int c = 0; c < kNK / 4; ++c)
          *reinterpret_cast<float4*>(stg + xoff(lane, c)) =
              make_float4(s[4 * c], s[4 * c + 1], s[4 * c + 2], s[4 * c + 3]);
        fence_async_smem();
        __syncwarp();
        if (lane == 0) {
          if (k >= 1 && !mbar_wait<true>(&bar->x_empty[xw], (k - 1) & 1, guard)) ok = false;
          if (ok) {
            bulk_copy_to_peer(x_remote, smem_u32(stg), kXWarp, xfull_remote);
            bulk_commit();
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        release_stage(t + ubase);   // as soon as the copy has read the slot
        // the peer's half of the same tile
        if (lane == 0) mbar_arrive_expect_tx(&bar->x_full[xw], kXWarp);
        if (!warp_wait<true>(&bar->x_full[xw], k & 1, guard)) { ok = false; break; }
#pragma unroll
        for (int c = 0; c < kNK / 4; ++c) {
          const float4 x = *reinterpret_cast<const float4*>(xslot + xoff(lane, c));
          s[4 * c] += x.x;
          s[4 * c + 1] += x.y;
          s[4 * c + 2] += x.z;
          s[4 * c + 3] += x.w;
        }
        // every lane has consumed its loads from the slot before lane 0 lets the peer refill it
        consume32(s);
        __syncwarp();
        if (grp == 1 && j + kGroups >= ntiles) xe_held = true;   // released after the epilogue
        else if (lane == 0) mbar_arrive_remote_relaxed(xempty_remote);
        const int key0 = k0 + j * kNK;
        const int nvalid = min(kNK, k1 - key0);
        if (p.logits && rank == 0 && h < p.n_heads && key0 >= 0 && !p.topk_idx) {
          float* lg =
              p.logits + (static_cast<size_t>(row) * p.n_heads + h) * p.max_seq_len + key0;
#pragma unroll
          for (int i = 0; i < kNK; ++i)
            if (i < nvalid && key0 + i < p.max_seq_len) lg[i] = s[i] * p.scale;
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
        // running-max decision for tile t (after another group decided tile t-1)
        float m_prev = -INFINITY;
        if (j > 0) {
          bool seen = true;
          if (seq[h] != t - 1) {
            const unsigned long long t0 = globaltimer_ns();
            uint32_t n = 0;
            while (seq[h] != t - 1) {
              if ((++n & 63u) == 0 &&
                  (guard.aborted() || globaltimer_ns() - t0 > guard.limit_ns)) {
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
          if (!warp_wait(&bar->pv_done[(t - 1) % kNB], ((t - 1) / kNB) & 1, guard)) {
            ok = false;
            break;
          }
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
#pragma unroll
        for (int i = 0; i < kNK; ++i) s[i] = fast_exp2(fmaf(s[i], c2, -m_dec));
#pragma unroll
        for (int i = 0; i < kNK / 2; ++i) pk[i] = pack_bf16x2(s[2 * i], s[2 * i + 1]);
#pragma unroll
        for (int i = 0; i < 16; ++i) s[i] += s[i + 16];
#pragma unroll
        for (int i = 0; i < 8; ++i) s[i] += s[i + 8];
#pragma unroll
        for (int i = 0; i < 4; ++i) s[i] += s[i + 4];
        l_g += (s[0] + s[2]) + (s[1] + s[3]);
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
      // final maximum of the row (decided at the last tile), all groups' sums relative to it
      {
        bool seen = true;
        const unsigned long long t0 = globaltimer_ns();
        uint32_t n = 0;
        while (seq[h] != glast) {
          if ((++n & 63u) == 0 && (guard.aborted() || globaltimer_ns() - t0 > guard.limit_ns)) {
            if (!guard.aborted()) guard.fail(kDevTimeout);
            seen = false;
            break;
          }
        }
        if (!__all_sync(0xffffffffu, seen)) break;
      }
      __threadfence_block();
      const float m_fin = m_ref[h];
      // (double-buffered by piece: a group cannot pass the next piece's sync_all before every
      // group has read this piece's sums)
      float* lsum = lsum_x + (pc & 1) * kGroups * 128;
      lsum[grp * 128 + h] = (m_used == -INFINITY) ? 0.f : l_g * fast_exp2(m_used - m_fin);
      if (!sync_all()) break;
      float l_tot = 0.f;
#pragma unroll
      for (int G = 0; G < kGroups; ++G) l_tot += lsum[G * 128 + h];
      const float inv_l = 1.f / l_tot;
      const float lse = (m_fin + log2f(l_tot)) * 0.69314718055994531f;
      const int slot = first_row ? 0 : 1;
      if (grp < 2) {
        // Groups 0 and 1 write the CTA's 256 columns of O (128 each) in blocks of 32 rows x 64
        // columns (bf16 for an uncut row, fp16 normalised partials for a cut one: 128-byte rows),
        // staged in the 128-byte-swizzle layout (lane = row, chunk c at c ^ (row & 7)), one TMA
        // tile store per block; the warps do not wait for the global writes.
        if (!warp_wait(&bar->pv_done[glast % kNB], (glast / kNB) & 1, guard)) break;
        tc_fence_after();
        const int ocol = col0 + grp * 128;
        const bool own_slot = (grp == 1 && xe_held);
        uint8_t* est = own_slot ? xslot : stg;
        const int u0 = g + ubase + grp * nblk;   // shared-slot uses (group 1: only if queued)
#pragma unroll 1
        for (int blk = 0; blk < nblk; ++blk) {
          uint32_t w[32];
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            float v[32];
            tmem_ld32(tmem + lane_off + kTmemO + grp * 128 + blk * 64 + half * 32, v);
#pragma unroll
            for (int i = 0; i < 16; ++i)
              w[16 * half + i] = whole ? pack_bf16x2(v[2 * i] * inv_l, v[2 * i + 1] * inv_l)
                                       : pack_f16x2(v[2 * i] * inv_l, v[2 * i + 1] * inv_l);
          }
          if (blk == nblk - 1) {   // every TMEM read of O is done: the next piece may overwrite it
            tc_fence_before();
            mbar_arrive(&bar->o_empty);
          }
          if (own_slot) {
            if (lane == 0) bulk_wait_read_all();
            __syncwarp();
          } else if (!acquire_stage(u0 + blk)) {
            ok = false;
            break;
          }
#pragma unroll
          for (int c = 0; c < 8; ++c)
            *reinterpret_cast<uint4*>(est + lane * 128 + ((c ^ (lane & 7)) << 4)) =
                make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
          fence_async_smem();
          __syncwarp();
          if (lane == 0) {
            if (whole) {
              if (quad * 32 < p.n_heads) tma_store_3d(&tmO, est, ocol + blk * 64, quad * 32, row);
            } else {
              tma_store_2d(&tmPart, est, ocol + blk * 64, (pair * 2 + slot) * 128 + quad * 32);
            }
            bulk_commit();
          }
          if (!own_slot) release_stage(u0 + blk);
        }
        if (!ok) break;
        if (own_slot) {   // the stores have read the slot: the peer may refill it
          if (lane == 0) {
            bulk_wait_read_all();
            mbar_arrive_remote_relaxed(xempty_remote);
          }
          xe_held = false;
        }
      } else {
        mbar_arrive(&bar->o_empty);   // this group reads no O
      }
      if (whole) {
        if (rank == 0 && grp == 0 && p.lse_out && h < p.n_heads)
          p.lse_out[static_cast<size_t>(row) * p.n_heads + h] = lse;
      } else if (rank == 0 && grp == 0) {
        p.part_lse[(static_cast<size_t>(pair) * 2 + slot) * 128 + h] = lse;
      }
      ubase += g1_has_tile ? nblk : 2 * nblk;
      ++pc;
      it.next();
    }
    if (lane == 0) bulk_wait_all();   // every copy and store this warp issued has completed
  }

  // ------------------------------------------------------------------ teardown
  if (warp == 1) {
    int dummy = 0;
    Guard drain{reinterpret_cast<volatile int*>(&dummy), p.status};
    mbar_wait(&bar->drain, 0, drain);   // every MMA this CTA issued has completed
  }
  tc_fence_before();
  __syncthreads();
  if (guard.aborted()) {   // every role has stopped: let the loads this thread armed land
    int dummy = 0;
    Guard drain{reinterpret_cast<volatile int*>(&dummy), p.status};
    for (int s = 0; s < kStages; ++s)
      if (last_slot[s] >= 0) mbar_wait(&bar->kv_full[s], (last_slot[s] / kStages) & 1, drain);
    if (qpe_armed > 0) mbar_wait(&bar->qpe_full, (qpe_armed - 1) & 1, drain);
  }
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
  return cudaLaunchKernelEx(&lc.cfg, latent_attention_kernel, m.kv, m.pe, m.q, m.qpe, m.o, m.part,
                            p.topk_idx ? m.kv2 : m.kv, p.topk_idx ? m.pe2 : m.pe, p);
}

bool make_gather_maps(AttnMaps* m, const void* kv, int64_t kv_sb, int64_t kv_st, const void* pe,
                      int64_t pe_sb, int64_t pe_st, int batch) {
  if (kv_sb % kv_st != 0 || pe_sb % pe_st != 0 || kv_sb / kv_st != pe_sb / pe_st) return false;
  const uint64_t rows = static_cast<uint64_t>(batch) * static_cast<uint64_t>(kv_sb / kv_st);
  if (rows >= (1ull << 31)) return false;   // gather row coordinates are 32-bit
  const uint64_t d_kv[2] = {kC, rows}, s_kv[1] = {static_cast<uint64_t>(kv_st) * 2};
  const uint64_t d_pe[2] = {kDr, rows}, s_pe[1] = {static_cast<uint64_t>(pe_st) * 2};
  const uint32_t box[2] = {64, 1}, box_pe[2] = {32, 1};
  return encode_tiled(&m->kv2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, kv, d_kv, s_kv, box,
                      CU_TENSOR_MAP_SWIZZLE_128B) &&
         encode_tiled(&m->pe2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, pe, d_pe, s_pe, box_pe,
                      CU_TENSOR_MAP_SWIZZLE_64B);
}

bool make_attention_maps(AttnMaps* m, const void* kv, int64_t kv_sb, int64_t kv_st, const void* pe,
                         int64_t pe_sb, int64_t pe_st, int batch, int max_seq_len, const void* qabs,
                         int rows, const void* o_lat, int n_heads, const void* part_o, int pairs) {
  const CUtensorMapDataType bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const CUtensorMapSwizzle sw = CU_TENSOR_MAP_SWIZZLE_128B;
  const uint64_t L = static_cast<uint64_t>(max_seq_len), Bt = static_cast<uint64_t>(batch);
  const uint64_t R = static_cast<uint64_t>(rows), H = static_cast<uint64_t>(n_heads);
  const uint32_t box_kv[3] = {64, static_cast<uint32_t>(kNK), 1};
  const uint32_t box_pe[3] = {32, static_cast<uint32_t>(kNK), 1};   // 64-byte rows
  const uint64_t d_kv[3] = {kC, L, Bt}, s_kv[2] = {static_cast<uint64_t>(kv_st) * 2,
                                                   static_cast<uint64_t>(kv_sb) * 2};
  const uint64_t d_pe[3] = {kDr, L, Bt}, s_pe[2] = {static_cast<uint64_t>(pe_st) * 2,
                                                    static_cast<uint64_t>(pe_sb) * 2};
  const uint64_t d_q[3] = {kDk, kHPad, R}, s_q[2] = {kDk * 2, kHPad * kDk * 2};
  const uint32_t box_q[3] = {64, 128, 1}, box_qpe[3] = {32, 128, 1};
  const uint64_t d_o[3] = {kC, H, R}, s_o[2] = {kC * 2, H * kC * 2};
  const uint32_t box_o[3] = {64, 32, 1};
  const uint64_t d_p[2] = {kC, static_cast<uint64_t>(pairs) * 2 * 128}, s_p[1] = {kC * 2};
  const uint32_t box_p[2] = {64, 32};
  return encode_tiled(&m->kv, bf, 3, kv, d_kv, s_kv, box_kv, sw) &&
         encode_tiled(&m->pe, bf, 3, pe, d_pe, s_pe, box_pe, CU_TENSOR_MAP_SWIZZLE_64B) &&
         encode_tiled(&m->q, bf, 3, qabs, d_q, s_q, box_q, sw) &&
         encode_tiled(&m->qpe, bf, 3, qabs, d_q, s_q, box_qpe, CU_TENSOR_MAP_SWIZZLE_64B) &&
         encode_tiled(&m->o, bf, 3, o_lat, d_o, s_o, box_o, sw) &&
         encode_tiled(&m->part, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, part_o, d_p, s_p, box_p, sw);
}

// ------------------------------------------------------------------------------------------
// Combine: rows cut between pairs merge their normalised partials by log-sum-exp weights.
// One warp per (row, head) task; lane l owns columns l, l+32, ..., l+480.
// ------------------------------------------------------------------------------------------

// Persistent grid (one block per SM, launched once): each warp walks (row, head) tasks.  Most
// rows are uncut, so a warp first reads the piece records of its next 32 tasks at once (one per
// lane, one round trip), then merges only the tasks whose row was cut.
constexpr int kCombineThreads = 512;

__global__ void __launch_bounds__(kCombineThreads) combine_kernel(const CombineParams p) {
  pdl_launch_dependents();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const long long warps = static_cast<long long>(gridDim.x) * (kCombineThreads / 32);
  const long long ntasks = static_cast<long long>(p.rows) * p.n_heads;
  for (long long base = static_cast<long long>(blockIdx.x) * (kCombineThreads / 32) + (threadIdx.x >> 5);
       base < ntasks; base += 32 * warps) {
    // this lane's task of the batch: base + lane * warps
    const long long mine = base + lane * warps;
    int2 rec = make_int2(0, 0);
    bool cut = false;
    if (mine < ntasks) {
      rec = __ldcg(p.row_pieces + mine / p.n_heads);
      const int plo = rec.x >> 1, phi = rec.y;
      if (plo < 0 || phi < plo || phi >= p.n_pairs) {   // not a record the key prefix can produce
        atomicCAS(p.status, kDevOk, kDevBadArg);
      } else {
        cut = plo != phi;   // an uncut row was written by one pair
      }
    }
    unsigned todo = __ballot_sync(0xffffffffu, cut);
    while (todo) {
      const int src = __ffs(todo) - 1;
      todo &= todo - 1;
      const long long task = base + src * warps;
      const int r = static_cast<int>(task / p.n_heads), h = static_cast<int>(task - static_cast<long long>(r) * p.n_heads);
      const int rx = __shfl_sync(0xffffffffu, rec.x, src), ry = __shfl_sync(0xffffffffu, rec.y, src);
      const int plo = rx >> 1, phi = ry;
      const int slot_lo = rx & 1;   // the first piece is the tail of a pair begun in an earlier row
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
            const int slot = q == plo ? slot_lo : 0;
            const size_t pbase = (static_cast<size_t>(q) * 2 + slot) * 128 + h;
            lse[b] = __ldg(p.part_lse + pbase);
            const __half* psrc = p.part_o + pbase * kC;
#pragma unroll
            for (int i = 0; i < 16; ++i) v[b][i] = __half2float(psrc[lane + 32 * i]);
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
