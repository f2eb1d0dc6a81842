// api.cu — the C ABI (include/mla.h): argument validation, workspace layout, TMA tensor-map
// creation and the launch chain of one decode / prefill call.
//
// Launch chain (one stream, no host synchronisation):
//   1. rmsnorm_kernel     a1 (+ rotary table, + per-row key prefix)
//   2. gemm (wq_b)        a2 + a3 (RoPE in the epilogue) → q_nope, rotary half of the query
//   3. gemm (absorb)      a4 → latent half of the absorbed query (per head, batched)
//   4. latent_attention   a5–a7 over the cache, split over keys across SM pairs
//   5. combine            LSE merge of rows cut between SM pairs
//   6. gemm (W_UV)        a8 → out
#include <math.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <new>

#include "mla.h"
#include "internal.h"
#include "tc100.cuh"

using namespace mla;

namespace {

constexpr int kMaxStages = 8;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

}  // namespace

bool mla::encode_tiled(CUtensorMap* m, CUtensorMapDataType dt, int rank, const void* base,
                  const uint64_t* dims, const uint64_t* strides, const uint32_t* box,
                  CUtensorMapSwizzle swizzle) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || rank < 1 || rank > 5) return false;
  cuuint64_t d[5], st[4];
  cuuint32_t b[5], es[5];
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    b[i] = box[i];
    es[i] = 1;
    if (i + 1 < rank) st[i] = strides[i];
  }
  return fn(m, dt, static_cast<cuuint32_t>(rank), const_cast<void*>(base), d, st, b, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

namespace {

// 3-D bf16 tensor map with 128-byte swizzle; strides in bytes for dims 1 and 2.
bool make_map(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
              uint64_t s1, uint64_t s2, uint32_t b0, uint32_t b1, uint32_t b2) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {s1, s2};
  cuuint32_t box[3] = {b0, b1, b2};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D map of FP8 codes (bytes) without swizzle: the converter warps read the slabs linearly.
bool make_map_u8(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                 uint64_t s1, uint64_t s2, uint32_t b0, uint32_t b1, uint32_t b2) {
  const uint64_t dims[3] = {d0, d1, d2}, strides[2] = {s1, s2};
  const uint32_t box[3] = {b0, b1, b2};
  return encode_tiled(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, base, dims, strides, box,
                      CU_TENSOR_MAP_SWIZZLE_NONE);
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

struct Layout {
  size_t status, w_ukt, y, rope, q_nope, qabs, o_lat, part_o, part_lse, prefix, pair_row,
      row_pieces, c_kv, total;
};

int device_pairs() { return attention_pairs(); }

bool config_ok(const mla_config* c, mla_status* why) {
  if (!c) {
    *why = MLA_ERR_INVALID_ARG;
    return false;
  }
  if (c->q_lora_rank != kR || c->kv_lora_rank != kC || c->qk_nope_head_dim != kDn ||
      c->qk_rope_head_dim != kDr || c->v_head_dim != kDv || c->n_heads < 16 || c->n_heads > 128 ||
      c->n_heads % 16 != 0) {
    *why = MLA_ERR_UNSUPPORTED;
    return false;
  }
  if (c->max_rows < 1 || c->max_rows > (1 << 20) || c->max_seq_len < 64 ||
      c->max_seq_len > (1 << 24) || !(c->rms_eps >= 0.f) || !(c->rope_theta > 0.f) ||
      !(c->softmax_scale >= 0.f) || !isfinite(c->softmax_scale)) {
    *why = MLA_ERR_INVALID_ARG;
    return false;
  }
  return true;
}

Layout layout_of(const mla_config* c) {
  const size_t H = c->n_heads, rows = c->max_rows, pairs = device_pairs();
  Layout L;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = round_up(off + bytes, 256);
    return o;
  };
  L.status = take(256);
  L.w_ukt = take(H * kC * kDn * 2);
  L.y = take(rows * kR * 2);
  L.rope = take(rows * kRopePairs * sizeof(float2));
  L.q_nope = take(rows * H * kDn * 2);
  L.qabs = take(rows * kHPad * kDk * 2);
  L.o_lat = take(rows * H * kC * 2);
  L.part_o = take(pairs * 2 * 128 * kC * 2);
  L.part_lse = take(pairs * 2 * 128 * 4);
  L.prefix = take((rows + 1) * 8);
  L.pair_row = take(pairs * 4);
  L.row_pieces = take(rows * 8);
  L.c_kv = take(rows * kDk * 2);
  L.total = off;
  return L;
}

}  // namespace

struct mla_ctx {
  mla_config cfg;
  int device;
  float scale;
  const float* gamma;
  const bf16* wq_b;
  const bf16* wkv_b;
  uint8_t* ws;
  Layout L;
  int n_pairs;
  CUtensorMap tm_wq, tm_wukt, tm_wuv;
  bool timing;
  cudaEvent_t ev[kMaxStages + 1];
  const char* stage_name[kMaxStages];
  int n_stages;
  int last_rows;
  int last_launches;
  // cache producer (mla_attach_producer)
  int prod_dim;
  const float* kv_gain;
  CUtensorMap tm_wqa, tm_wkva;
  // FP8 block-scaled weights (mla_init_fp8): scales [H*192/128, 12] and [2H, 4]; null for bf16
  const float* wq_scale;
  const float* wkv_scale;
  unsigned long long gemm_wait_ns;   // mla_set_wait_limit (0: the kernels' 2 s default)

  int* status() const { return reinterpret_cast<int*>(ws + L.status); }
  bf16* w_ukt() const { return reinterpret_cast<bf16*>(ws + L.w_ukt); }
  bf16* y() const { return reinterpret_cast<bf16*>(ws + L.y); }
  float2* rope() const { return reinterpret_cast<float2*>(ws + L.rope); }
  bf16* q_nope() const { return reinterpret_cast<bf16*>(ws + L.q_nope); }
  bf16* qabs() const { return reinterpret_cast<bf16*>(ws + L.qabs); }
  bf16* o_lat() const { return reinterpret_cast<bf16*>(ws + L.o_lat); }
  __half* part_o() const { return reinterpret_cast<__half*>(ws + L.part_o); }
  float* part_lse() const { return reinterpret_cast<float*>(ws + L.part_lse); }
  long long* prefix() const { return reinterpret_cast<long long*>(ws + L.prefix); }
  int* pair_row() const { return reinterpret_cast<int*>(ws + L.pair_row); }
  int2* row_pieces() const { return reinterpret_cast<int2*>(ws + L.row_pieces); }
  bf16* c_kv() const { return reinterpret_cast<bf16*>(ws + L.c_kv); }
};

namespace {

// Records an event before stage `i` when timing is on.
struct StageClock {
  mla_ctx* c;
  cudaStream_t s;
  int n = 0;
  void mark(const char* name) {
    if (!c->timing) return;
    if (n < kMaxStages) {
      c->stage_name[n] = name;
      cudaEventRecord(c->ev[n], s);
    }
    ++n;
  }
  void finish() {
    if (!c->timing) return;
    const int k = n < kMaxStages ? n : kMaxStages;
    cudaEventRecord(c->ev[k], s);
    c->n_stages = k;
  }
};

mla_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MLA_OK : MLA_ERR_CUDA; }

// A launch that fails is reported on stderr with the kernel's name, then MLA_ERR_CUDA returns.
#define MLA_TRY(expr)                                                                       \
  do {                                                                                      \
    cudaError_t _e = (expr);                                                                \
    if (_e != cudaSuccess) {                                                                \
      fprintf(stderr, "mla: %s failed: %s\n", #expr, cudaGetErrorString(_e));             \
      return MLA_ERR_CUDA;                                                                  \
    }                                                                                       \
  } while (0)

// Index-mask decode: per row the selected keys (topk_idx [B, k], counts topk_len [B]).
struct Sparse {
  const int32_t* idx = nullptr;
  const int32_t* len = nullptr;
  int k = 0;
};

// The whole path for `rows` query rows.  decode: start_pos_dev != null, T = 1.
mla_status run_path(mla_ctx* c, const void* q_latent, void* residual, const int32_t* start_pos_dev,
                    int start_pos, int T, int B, const void* kv, int64_t kv_sb, int64_t kv_st,
                    const void* pe, int64_t pe_sb, int64_t pe_st, void* out, float* lse,
                    float* logits, cudaStream_t s, const Sparse& sp = Sparse()) {
  const int rows = B * T;
  const int H = c->cfg.n_heads;
  const int bn = gemm_bn(rows);
  StageClock clk{c, s};
  int launches = 0;

  // per-call tensor maps
  CUtensorMap tm_y, tm_qn, tm_olat;
  AttnMaps am;
  const uint64_t rws = static_cast<uint64_t>(rows);
  if (!make_map(&tm_y, c->y(), kR, 1, rws, kR * 2, kR * 2, 64, 1, bn) ||
      !make_map(&tm_qn, c->q_nope(), kDn, H, rws, kDn * 2, static_cast<uint64_t>(H) * kDn * 2, 64,
                1, bn) ||
      !make_map(&tm_olat, c->o_lat(), kC, H, rws, kC * 2, static_cast<uint64_t>(H) * kC * 2, 64, 1,
                bn) ||
      !make_attention_maps(&am, kv, kv_sb, kv_st, pe, pe_sb, pe_st, B, c->cfg.max_seq_len, c->qabs(),
                           rows, c->o_lat(), H, c->part_o(), c->n_pairs) ||
      (sp.idx && !make_gather_maps(&am, kv, kv_sb, kv_st, pe, pe_sb, pe_st, B)))
    return MLA_ERR_INVALID_ARG;

  // Kernels 2-6 are launched with programmatic dependent launch: each starts on SMs its
  // predecessor has released and waits (griddepcontrol.wait) before touching that kernel's data;
  // kernel 1 is an ordinary launch, so the chain starts after all earlier work of the stream.
  // 1. q_norm (+ residual), rotary table, key prefix
  RmsParams rp{};
  rp.x = static_cast<const bf16*>(q_latent);
  rp.residual = static_cast<bf16*>(residual);
  rp.gamma = c->gamma;
  rp.y = c->y();
  rp.rows = rows;
  rp.dim = kR;
  rp.eps = c->cfg.rms_eps;
  rp.rope_tab = c->rope();
  rp.rope_log_theta = log(static_cast<double>(c->cfg.rope_theta));
  rp.start_pos_dev = start_pos_dev;
  rp.start_pos = start_pos;
  rp.T = T;
  rp.max_seq_len = c->cfg.max_seq_len;
  rp.row_prefix = c->prefix();
  rp.pair_row = c->pair_row();
  rp.row_pieces = c->row_pieces();
  rp.n_pairs = c->n_pairs;
  rp.min_keys_per_pair = kMinKeysPerPair;
  rp.status = c->status();
  rp.topk_len = sp.len;
  rp.topk_k = sp.k;
  clk.mark("rmsnorm");
  MLA_TRY(launch_rmsnorm(rp, s));
  ++launches;

  // 2. wq_b + RoPE
  GemmParams g1{};
  g1.M = H * kDq;
  g1.N = rows;
  g1.K = kR;
  g1.epi = kEpiWqbRope;
  g1.out0 = c->q_nope();
  g1.ld_n0 = static_cast<long long>(H) * kDn;
  g1.out1 = c->qabs();
  g1.rope_tab = c->rope();
  g1.n_heads = H;
  g1.status = c->status();
  if (c->wq_scale) {   // 128 x 128 blocks of wq_b [H*192, 1536]
    g1.a_scale = c->wq_scale;
    g1.a_sm = kR / 128;
    g1.a_sk = 1;
    g1.a_scale_n = static_cast<long long>(H) * kDq / 128 * (kR / 128);
  }
  clk.mark("wq_b_rope");
  g1.wait_limit_ns = c->gemm_wait_ns;
  MLA_TRY(launch_gemm(c->tm_wq, tm_y, g1, 1, s, true));
  ++launches;

  // 3. W_UK absorption (one batch per head)
  GemmParams g2{};
  g2.M = kC;
  g2.N = rows;
  g2.K = kDn;
  g2.epi = kEpiStore;
  g2.out0 = c->qabs();
  g2.ld_n0 = static_cast<long long>(kHPad) * kDk;
  g2.ld_g0 = kDk;
  g2.n_heads = H;
  g2.status = c->status();
  if (c->wkv_scale) {   // W_UK^T[h] row block c/128 = block (2h, c/128) of wkv_b [H*256, 512]
    g2.a_scale = c->wkv_scale;
    g2.a_sg = 2 * (kC / 128);
    g2.a_sm = 1;
    g2.a_sk = 0;
    g2.a_scale_n = static_cast<long long>(H) * 2 * (kC / 128);
  }
  clk.mark("absorb_w_uk");
  g2.wait_limit_ns = c->gemm_wait_ns;
  MLA_TRY(launch_gemm(c->tm_wukt, tm_qn, g2, H, s, true));
  ++launches;

  // 4. latent attention
  AttnParams ap{};
  ap.row_prefix = c->prefix();
  ap.qabs = c->qabs();
  ap.rows = rows;
  ap.T = T;
  ap.n_heads = H;
  ap.scale = c->scale;
  ap.scale_log2 = c->scale * 1.4426950408889634f;
  ap.min_keys_per_pair = kMinKeysPerPair;
  ap.o_lat = c->o_lat();
  ap.lse_out = lse;
  ap.logits = logits;
  ap.max_seq_len = c->cfg.max_seq_len;
  ap.part_o = c->part_o();
  ap.part_lse = c->part_lse();
  ap.pair_row = c->pair_row();
  ap.status = c->status();
  ap.topk_idx = sp.idx;
  ap.topk_k = sp.k;
  ap.seq_rows = sp.idx ? kv_sb / kv_st : 0;
  clk.mark("latent_attention");
  MLA_TRY(launch_attention(am, ap, c->n_pairs, s, true));
  ++launches;

  // 5. combine rows cut between pairs — for at most 64 rows the W_UV GEMM merges them itself
  // while it builds its B operand (no separate launch)
  const bool merge_in_wuv = rows <= 64;
  CombineParams cp{};
  cp.row_prefix = c->prefix();
  cp.rows = rows;
  cp.n_heads = H;
  cp.n_pairs = c->n_pairs;
  cp.min_keys_per_pair = kMinKeysPerPair;
  cp.part_o = c->part_o();
  cp.part_lse = c->part_lse();
  cp.row_pieces = c->row_pieces();
  cp.o_lat = c->o_lat();
  cp.lse_out = lse;
  cp.status = c->status();
  if (!merge_in_wuv) {
    clk.mark("combine");
    MLA_TRY(launch_combine(cp, s, true));
    ++launches;
  }

  // 6. W_UV expansion (one batch per head)
  GemmParams g3{};
  g3.M = kDv;
  g3.N = rows;
  g3.K = kC;
  g3.a_row_off = kDn;
  g3.epi = kEpiStore;
  g3.out0 = static_cast<bf16*>(out);
  g3.ld_n0 = static_cast<long long>(H) * kDv;
  g3.ld_g0 = kDv;
  g3.n_heads = H;
  g3.status = c->status();
  if (c->wkv_scale) {   // W_UV[h] = block row 2h+1 of wkv_b (a_row_off = 128 selects it)
    g3.a_scale = c->wkv_scale;
    g3.a_sg = 2 * (kC / 128);
    g3.a_sm = kC / 128;
    g3.a_sk = 1;
    g3.a_scale_n = static_cast<long long>(H) * 2 * (kC / 128);
  }
  if (merge_in_wuv) {
    g3.bmerge = 1;
    g3.row_prefix = c->prefix();
    g3.part_o = c->part_o();
    g3.part_lse = c->part_lse();
    g3.row_pieces = c->row_pieces();
    g3.o_lat = c->o_lat();
    g3.lse_out = lse;
    g3.n_pairs = c->n_pairs;
    g3.min_keys_per_pair = kMinKeysPerPair;
  }
  clk.mark("w_uv");
  g3.wait_limit_ns = c->gemm_wait_ns;
  MLA_TRY(launch_gemm(c->tm_wuv, tm_olat, g3, H, s, true));
  ++launches;
  clk.finish();

  c->last_rows = rows;
  c->last_launches = launches;
  return MLA_OK;
}

// The prefill chunk in the non-absorbed form: q_norm → wq_b + RoPE (as the absorbed path) →
// per sequence, keys and values rebuilt from the latent (one GEMM: kvb = kv · wkv_b^T) →
// multi-head attention with the causal mask → optionally wo.
mla_status run_mha(mla_ctx* c, const void* q_latent, void* residual, int start_pos, int T, int B,
                   const void* kv, int64_t kv_sb, int64_t kv_st, const void* pe, int64_t pe_sb,
                   int64_t pe_st, void* kvb, void* out, float* lse, const void* wo, int dim,
                   void* y, cudaStream_t s) {
  const int rows = B * T;
  const int H = c->cfg.n_heads;
  const int Lk = start_pos + T;
  StageClock clk{c, s};
  int launches = 0;
  const uint64_t rws = static_cast<uint64_t>(rows);
  CUtensorMap tm_y, tm_out, tm_wo;
  FmhaMaps fm;
  const uint64_t kvb_row = static_cast<uint64_t>(H) * 256;   // elements per rebuilt key row
  if (!make_map(&tm_y, c->y(), kR, 1, rws, kR * 2, kR * 2, 64, 1, gemm_bn(rows)) ||
      !make_map(&fm.qn, c->q_nope(), kDn, H, rws, kDn * 2, static_cast<uint64_t>(H) * kDn * 2, 64,
                1, 128) ||
      !make_map(&fm.qp, c->qabs(), kDk, kHPad, rws, kDk * 2, static_cast<uint64_t>(kHPad) * kDk * 2,
                64, 1, 128) ||
      !make_map(&fm.kvb, kvb, kvb_row, static_cast<uint64_t>(Lk), static_cast<uint64_t>(B),
                kvb_row * 2, kvb_row * Lk * 2, 64, 128, 1) ||
      !make_map(&fm.pe, pe, kDr, static_cast<uint64_t>(c->cfg.max_seq_len),
                static_cast<uint64_t>(B), static_cast<uint64_t>(pe_st) * 2,
                static_cast<uint64_t>(pe_sb) * 2, 64, 128, 1))
    return MLA_ERR_INVALID_ARG;
  if (wo && (!make_map(&tm_out, out, static_cast<uint64_t>(H) * kDv, 1, rws,
                       static_cast<uint64_t>(H) * kDv * 2, static_cast<uint64_t>(H) * kDv * 2, 64,
                       1, gemm_bn(rows)) ||
             !make_map(&tm_wo, wo, static_cast<uint64_t>(H) * kDv, static_cast<uint64_t>(dim), 1,
                       static_cast<uint64_t>(H) * kDv * 2,
                       static_cast<uint64_t>(H) * kDv * 2 * dim, 64, 128, 1)))
    return MLA_ERR_INVALID_ARG;

  RmsParams rp{};
  rp.x = static_cast<const bf16*>(q_latent);
  rp.residual = static_cast<bf16*>(residual);
  rp.gamma = c->gamma;
  rp.y = c->y();
  rp.rows = rows;
  rp.dim = kR;
  rp.eps = c->cfg.rms_eps;
  rp.rope_tab = c->rope();
  rp.rope_log_theta = log(static_cast<double>(c->cfg.rope_theta));
  rp.start_pos = start_pos;
  rp.T = T;
  rp.max_seq_len = c->cfg.max_seq_len;
  rp.status = c->status();
  clk.mark("rmsnorm");
  MLA_TRY(launch_rmsnorm(rp, s));
  ++launches;

  GemmParams g1{};
  g1.M = H * kDq;
  g1.N = rows;
  g1.K = kR;
  g1.epi = kEpiWqbRope;
  g1.out0 = c->q_nope();
  g1.ld_n0 = static_cast<long long>(H) * kDn;
  g1.out1 = c->qabs();
  g1.rope_tab = c->rope();
  g1.n_heads = H;
  g1.status = c->status();
  clk.mark("wq_b_rope");
  g1.wait_limit_ns = c->gemm_wait_ns;
  MLA_TRY(launch_gemm(c->tm_wq, tm_y, g1, 1, s, true));
  ++launches;

  // keys and values of every head from the latent: kvb[b][key][h*256 + j] = wkv_b[h*256+j] · kv
  clk.mark("kv_rebuild");
  for (int b = 0; b < B; ++b) {
    CUtensorMap tm_kv;
    const bf16* kvb_src = static_cast<const bf16*>(kv) + static_cast<size_t>(b) * kv_sb;
    if (!make_map(&tm_kv, kvb_src, kC, 1, static_cast<uint64_t>(Lk),
                  static_cast<uint64_t>(kv_st) * 2, static_cast<uint64_t>(kv_st) * 2, 64, 1,
                  gemm_bn(Lk)))
      return MLA_ERR_INVALID_ARG;
    GemmParams gk{};
    gk.M = kDn + kDv;
    gk.N = Lk;
    gk.K = kC;
    gk.epi = kEpiStore;
    gk.out0 = static_cast<bf16*>(kvb) + static_cast<size_t>(b) * Lk * kvb_row;
    gk.ld_n0 = static_cast<long long>(kvb_row);
    gk.ld_g0 = kDn + kDv;
    gk.n_heads = H;
    gk.status = c->status();
    gk.b_g0 = 1;
    gk.wait_limit_ns = c->gemm_wait_ns;
    MLA_TRY(launch_gemm(c->tm_wuv, tm_kv, gk, H, s, true));
    ++launches;
  }

  FmhaParams fp{};
  fp.out = static_cast<bf16*>(out);
  fp.lse = lse;
  fp.T = T;
  fp.B = B;
  fp.n_heads = H;
  fp.start_pos = start_pos;
  fp.scale_log2 = c->scale * 1.4426950408889634f;
  fp.status = c->status();
  clk.mark("mha");
  MLA_TRY(launch_fmha(fm, fp, s, true));
  ++launches;

  if (wo) {
    GemmParams go{};
    go.M = dim;
    go.N = rows;
    go.K = H * kDv;
    go.epi = kEpiStore;
    go.out0 = static_cast<bf16*>(y);
    go.ld_n0 = dim;
    go.n_heads = H;
    go.status = c->status();
    clk.mark("wo");
    go.wait_limit_ns = c->gemm_wait_ns;
    MLA_TRY(launch_gemm(tm_wo, tm_out, go, 1, s, true));
    ++launches;
  }
  clk.finish();
  c->last_rows = rows;
  c->last_launches = launches;
  return MLA_OK;
}

// Cache producer for `rows` = B*T new tokens: q_latent = x wq_a^T; c = x wkv_a^T → kv_norm /
// key RoPE → the tokens' cache rows.
mla_status run_produce(mla_ctx* c, const void* x, const int32_t* start_pos_dev, int start_pos,
                       int T, int B, void* kv, int64_t kv_sb, int64_t kv_st, void* pe,
                       int64_t pe_sb, int64_t pe_st, void* q_latent, cudaStream_t s) {
  const int rows = B * T;
  const int bn = gemm_bn(rows);
  StageClock clk{c, s};
  CUtensorMap tm_x;
  const uint64_t dim = static_cast<uint64_t>(c->prod_dim);
  if (!make_map(&tm_x, x, dim, 1, static_cast<uint64_t>(rows), dim * 2, dim * 2, 64, 1, bn))
    return MLA_ERR_INVALID_ARG;
  GemmParams gq{};
  gq.M = kR;
  gq.N = rows;
  gq.K = c->prod_dim;
  gq.epi = kEpiStore;
  gq.out0 = static_cast<bf16*>(q_latent);
  gq.ld_n0 = kR;
  gq.status = c->status();
  clk.mark("wq_a");
  gq.wait_limit_ns = c->gemm_wait_ns;
  MLA_TRY(launch_gemm(c->tm_wqa, tm_x, gq, 1, s, false));
  GemmParams gk{};
  gk.M = kDk;   // 576 = 4.5 weight tiles: the last tile's upper half reads zero rows
  gk.N = rows;
  gk.K = c->prod_dim;
  gk.epi = kEpiStore;
  gk.out0 = c->c_kv();
  gk.ld_n0 = kDk;
  gk.status = c->status();
  clk.mark("wkv_a");
  gk.wait_limit_ns = c->gemm_wait_ns;
  MLA_TRY(launch_gemm(c->tm_wkva, tm_x, gk, 1, s, true));
  KvFinishParams kp{};
  kp.c = c->c_kv();
  kp.gain = c->kv_gain;
  kp.kv_cache = static_cast<bf16*>(kv);
  kp.kv_sb = kv_sb;
  kp.kv_st = kv_st;
  kp.pe_cache = static_cast<bf16*>(pe);
  kp.pe_sb = pe_sb;
  kp.pe_st = pe_st;
  kp.rows = rows;
  kp.T = T;
  kp.start_pos_dev = start_pos_dev;
  kp.start_pos = start_pos;
  kp.max_seq_len = c->cfg.max_seq_len;
  kp.eps = c->cfg.rms_eps;
  kp.rope_log_theta = log(static_cast<double>(c->cfg.rope_theta));
  kp.status = c->status();
  clk.mark("kv_finish");
  MLA_TRY(launch_kv_finish(kp, s, true));
  clk.finish();
  c->last_launches = 3;
  return MLA_OK;
}

}  // namespace

extern "C" {

const char* mla_status_string(mla_status s) {
  switch (s) {
    case MLA_OK: return "MLA_OK";
    case MLA_ERR_INVALID_ARG: return "MLA_ERR_INVALID_ARG";
    case MLA_ERR_UNSUPPORTED: return "MLA_ERR_UNSUPPORTED";
    case MLA_ERR_WORKSPACE: return "MLA_ERR_WORKSPACE";
    case MLA_ERR_CUDA: return "MLA_ERR_CUDA";
    case MLA_ERR_DEVICE_TIMEOUT: return "MLA_ERR_DEVICE_TIMEOUT";
    case MLA_ERR_DEVICE_ARG: return "MLA_ERR_DEVICE_ARG";
  }
  return "MLA_ERR_UNKNOWN";
}

size_t mla_workspace_size(const mla_config* cfg) {
  mla_status why;
  if (!config_ok(cfg, &why)) return 0;
  return layout_of(cfg).total;
}

}  // extern "C"

namespace {

// Shared set-up of mla_init / mla_init_fp8.  fp8: the weights are E4M3 codes (one byte each)
// with 128 x 128 block scales; the tensor maps read bytes and W_UK^T is copied as bytes.
mla_status init_ctx(const mla_config* cfg, const float* q_norm_gain, const void* wq_b,
                    const void* wkv_b, const float* wq_scale, const float* wkv_scale,
                    void* workspace, size_t workspace_bytes, cudaStream_t stream, mla_ctx** out) {
  const bool fp8 = wq_scale != nullptr;
  if (!out) return MLA_ERR_INVALID_ARG;
  *out = nullptr;
  mla_status why;
  if (!config_ok(cfg, &why)) return why;
  if (!q_norm_gain || !wq_b || !wkv_b || !aligned(q_norm_gain, 16) || !aligned(wq_b, 16) ||
      !aligned(wkv_b, 16))
    return MLA_ERR_INVALID_ARG;
  const Layout L = layout_of(cfg);
  if (!workspace || !aligned(workspace, 256) || workspace_bytes < L.total) return MLA_ERR_WORKSPACE;

  static unsigned long long prepared = 0;   // kernel attributes are set once per device
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return MLA_ERR_CUDA;
  if (!(prepared & (1ull << dev))) {
    if (gemm_prepare() != cudaSuccess || attention_prepare() != cudaSuccess ||
        fmha_prepare() != cudaSuccess)
      return MLA_ERR_CUDA;
    prepared |= 1ull << dev;
  }

  mla_ctx* c = new (std::nothrow) mla_ctx();
  if (!c) return MLA_ERR_CUDA;
  c->cfg = *cfg;
  c->device = dev;
  c->scale = cfg->softmax_scale > 0.f
                 ? cfg->softmax_scale
                 : static_cast<float>(1.0 / sqrt(static_cast<double>(kDn + kDr)));
  c->gamma = q_norm_gain;
  c->wq_b = static_cast<const bf16*>(wq_b);
  c->wkv_b = static_cast<const bf16*>(wkv_b);
  c->ws = static_cast<uint8_t*>(workspace);
  c->L = L;
  c->n_pairs = device_pairs();
  c->timing = false;
  c->n_stages = 0;
  c->last_rows = 0;
  c->last_launches = 0;
  c->prod_dim = 0;
  c->kv_gain = nullptr;
  c->wq_scale = wq_scale;
  c->wkv_scale = wkv_scale;
  c->gemm_wait_ns = 0;
  for (int i = 0; i <= kMaxStages; ++i) c->ev[i] = nullptr;

  const int H = cfg->n_heads;
  const uint64_t e = fp8 ? 1 : 2;   // bytes per weight element
  uint8_t* wukt = reinterpret_cast<uint8_t*>(c->w_ukt());
  auto map = fp8 ? make_map_u8 : make_map;
  bool ok = map(&c->tm_wq, wq_b, kR, static_cast<uint64_t>(H) * kDq, 1, kR * e,
                static_cast<uint64_t>(H) * kDq * kR * e, 64, 128, 1) &&
            map(&c->tm_wukt, wukt, kDn, kC, H, kDn * e, static_cast<uint64_t>(kC) * kDn * e, 64,
                128, 1) &&
            map(&c->tm_wuv, wkv_b, kC, kDn + kDv, H, kC * e,
                static_cast<uint64_t>(kDn + kDv) * kC * e, 64, 128, 1);
  if (!ok) {
    delete c;
    return MLA_ERR_CUDA;
  }
  // zero the workspace first (stream order), then the one-time W_UK^T copy into it
  if (cudaMemsetAsync(workspace, 0, L.total, stream) != cudaSuccess ||
      (fp8 ? launch_transpose_uk_fp8(static_cast<const uint8_t*>(wkv_b), wukt, H, stream)
           : launch_transpose_uk(c->wkv_b, c->w_ukt(), H, stream)) != cudaSuccess) {
    delete c;
    return MLA_ERR_CUDA;
  }
  *out = c;
  return MLA_OK;
}

}  // namespace

extern "C" {

mla_status mla_init(const mla_config* cfg, const float* q_norm_gain, const void* wq_b,
                    const void* wkv_b, void* workspace, size_t workspace_bytes, cudaStream_t stream,
                    mla_ctx** out) {
  return init_ctx(cfg, q_norm_gain, wq_b, wkv_b, nullptr, nullptr, workspace, workspace_bytes,
                  stream, out);
}

mla_status mla_init_fp8(const mla_config* cfg, const float* q_norm_gain, const void* wq_b_fp8,
                        const float* wq_b_scale, const void* wkv_b_fp8, const float* wkv_b_scale,
                        void* workspace, size_t workspace_bytes, cudaStream_t stream,
                        mla_ctx** out) {
  if (!out) return MLA_ERR_INVALID_ARG;
  *out = nullptr;
  if (!wq_b_scale || !wkv_b_scale || !aligned(wq_b_scale, 4) || !aligned(wkv_b_scale, 4))
    return MLA_ERR_INVALID_ARG;
  return init_ctx(cfg, q_norm_gain, wq_b_fp8, wkv_b_fp8, wq_b_scale, wkv_b_scale, workspace,
                  workspace_bytes, stream, out);
}

void mla_destroy(mla_ctx* ctx) {
  if (!ctx) return;
  for (int i = 0; i <= kMaxStages; ++i)
    if (ctx->ev[i]) cudaEventDestroy(ctx->ev[i]);
  delete ctx;
}

mla_status mla_rmsnorm(const void* x, void* residual, const float* gain, int32_t rows, int32_t dim,
                       float eps, void* y, cudaStream_t stream) {
  if (!x || !gain || !y || rows < 1 || dim < 256 || dim > 4096 || dim % 256 != 0 ||
      !(eps >= 0.f))
    return MLA_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(y, 16) || !aligned(gain, 16) ||
      (residual && !aligned(residual, 16)) || x == y)
    return MLA_ERR_INVALID_ARG;
  RmsParams rp{};
  rp.x = static_cast<const bf16*>(x);
  rp.residual = static_cast<bf16*>(residual);
  rp.gamma = gain;
  rp.y = static_cast<bf16*>(y);
  rp.rows = rows;
  rp.dim = dim;
  rp.eps = eps;
  rp.T = 1;
  rp.max_seq_len = 1;
  return cuda_status(launch_rmsnorm(rp, stream));
}

mla_status mla_decode(mla_ctx* ctx, const void* q_latent, void* residual, const int32_t* start_pos,
                      const void* kv_cache, int64_t kv_stride_b, int64_t kv_stride_t,
                      const void* pe_cache, int64_t pe_stride_b, int64_t pe_stride_t, int32_t B,
                      void* out, float* lse, float* logits, cudaStream_t stream) {
  if (!ctx || !q_latent || !start_pos || !out) return MLA_ERR_INVALID_ARG;
  if (B < 1 || B > ctx->cfg.max_rows) return MLA_ERR_INVALID_ARG;
  if (!aligned(q_latent, 16) || !aligned(out, 16) || !aligned(start_pos, 4) ||
      (residual && !aligned(residual, 16)) || (lse && !aligned(lse, 4)) ||
      (logits && !aligned(logits, 4)))
    return MLA_ERR_INVALID_ARG;
  if (!cache_args_ok(kv_cache, kv_stride_b, kv_stride_t, pe_cache, pe_stride_b, pe_stride_t))
    return MLA_ERR_INVALID_ARG;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev != ctx->device) return MLA_ERR_INVALID_ARG;
  return run_path(ctx, q_latent, residual, start_pos, 0, 1, B, kv_cache, kv_stride_b, kv_stride_t,
                  pe_cache, pe_stride_b, pe_stride_t, out, lse, logits, stream);
}

mla_status mla_decode_sparse(mla_ctx* ctx, const void* q_latent, void* residual,
                             const int32_t* start_pos, const int32_t* topk_idx,
                             const int32_t* topk_len, int32_t k, const void* kv_cache,
                             int64_t kv_stride_b, int64_t kv_stride_t, const void* pe_cache,
                             int64_t pe_stride_b, int64_t pe_stride_t, int32_t B, void* out,
                             float* lse, cudaStream_t stream) {
  if (!ctx || !q_latent || !start_pos || !topk_idx || !topk_len || !out) return MLA_ERR_INVALID_ARG;
  if (B < 1 || B > ctx->cfg.max_rows || k < 1 || k > (1 << 24)) return MLA_ERR_INVALID_ARG;
  if (!aligned(q_latent, 16) || !aligned(out, 16) || !aligned(start_pos, 4) ||
      !aligned(topk_idx, 4) || !aligned(topk_len, 4) || (residual && !aligned(residual, 16)) ||
      (lse && !aligned(lse, 4)))
    return MLA_ERR_INVALID_ARG;
  if (!cache_args_ok(kv_cache, kv_stride_b, kv_stride_t, pe_cache, pe_stride_b, pe_stride_t))
    return MLA_ERR_INVALID_ARG;
  if (kv_stride_b % kv_stride_t != 0 || pe_stride_b % pe_stride_t != 0 ||
      kv_stride_b / kv_stride_t != pe_stride_b / pe_stride_t)
    return MLA_ERR_INVALID_ARG;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev != ctx->device) return MLA_ERR_INVALID_ARG;
  Sparse sp;
  sp.idx = topk_idx;
  sp.len = topk_len;
  sp.k = k;
  return run_path(ctx, q_latent, residual, start_pos, 0, 1, B, kv_cache, kv_stride_b, kv_stride_t,
                  pe_cache, pe_stride_b, pe_stride_t, out, lse, nullptr, stream, sp);
}

mla_status mla_prefill_chunk(mla_ctx* ctx, const void* q_latent, void* residual, int32_t start_pos,
                             int32_t T, const void* kv_cache, int64_t kv_stride_b,
                             int64_t kv_stride_t, const void* pe_cache, int64_t pe_stride_b,
                             int64_t pe_stride_t, int32_t B, void* out, float* lse,
                             cudaStream_t stream) {
  if (!ctx || !q_latent || !out) return MLA_ERR_INVALID_ARG;
  if (B < 1 || T < 1 || static_cast<int64_t>(B) * T > ctx->cfg.max_rows || start_pos < 0 ||
      static_cast<int64_t>(start_pos) + T > ctx->cfg.max_seq_len)
    return MLA_ERR_INVALID_ARG;
  if (!aligned(q_latent, 16) || !aligned(out, 16) || (residual && !aligned(residual, 16)) ||
      (lse && !aligned(lse, 4)))
    return MLA_ERR_INVALID_ARG;
  if (!cache_args_ok(kv_cache, kv_stride_b, kv_stride_t, pe_cache, pe_stride_b, pe_stride_t))
    return MLA_ERR_INVALID_ARG;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev != ctx->device) return MLA_ERR_INVALID_ARG;
  return run_path(ctx, q_latent, residual, nullptr, start_pos, T, B, kv_cache, kv_stride_b,
                  kv_stride_t, pe_cache, pe_stride_b, pe_stride_t, out, lse, nullptr, stream);
}

mla_status mla_sync_status(mla_ctx* ctx, cudaStream_t stream) {
  if (!ctx) return MLA_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return MLA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, ctx->status(), sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return MLA_ERR_CUDA;
  if (v != 0 && cudaMemset(ctx->status(), 0, sizeof(int)) != cudaSuccess) return MLA_ERR_CUDA;
  if (v == kDevTimeout) return MLA_ERR_DEVICE_TIMEOUT;
  if (v == kDevBadArg) return MLA_ERR_DEVICE_ARG;
  return v == 0 ? MLA_OK : MLA_ERR_CUDA;
}

mla_status mla_enable_stage_timing(mla_ctx* ctx, int32_t enable) {
  if (!ctx) return MLA_ERR_INVALID_ARG;
  if (enable && !ctx->ev[0]) {
    for (int i = 0; i <= kMaxStages; ++i)
      if (cudaEventCreate(&ctx->ev[i]) != cudaSuccess) return MLA_ERR_CUDA;
  }
  ctx->timing = enable != 0;
  return MLA_OK;
}

mla_status mla_stage_times(mla_ctx* ctx, float* ms, const char** names, int32_t cap, int32_t* n) {
  if (!ctx || !n || cap < 0 || (cap > 0 && !ms)) return MLA_ERR_INVALID_ARG;
  *n = ctx->n_stages;
  if (!ctx->timing || ctx->n_stages == 0) return MLA_OK;
  if (cudaEventSynchronize(ctx->ev[ctx->n_stages]) != cudaSuccess) return MLA_ERR_CUDA;
  for (int i = 0; i < ctx->n_stages && i < cap; ++i) {
    if (cudaEventElapsedTime(&ms[i], ctx->ev[i], ctx->ev[i + 1]) != cudaSuccess) return MLA_ERR_CUDA;
    if (names) names[i] = ctx->stage_name[i];
  }
  return MLA_OK;
}

mla_status mla_debug_copy(mla_ctx* ctx, int32_t which, void* dst, size_t bytes,
                          cudaStream_t stream) {
  if (!ctx || !dst) return MLA_ERR_INVALID_ARG;
  const size_t rows = ctx->last_rows, H = ctx->cfg.n_heads;
  const void* src = nullptr;
  size_t cap = 0;
  switch (which) {
    case 0: src = ctx->y(); cap = rows * kR * 2; break;
    case 1: src = ctx->q_nope(); cap = rows * H * kDn * 2; break;
    case 2: src = ctx->qabs(); cap = rows * kHPad * kDk * 2; break;
    case 3: src = ctx->o_lat(); cap = rows * H * kC * 2; break;
    default: return MLA_ERR_INVALID_ARG;
  }
  if (bytes > cap) return MLA_ERR_INVALID_ARG;
  return cuda_status(cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToDevice, stream));
}

int32_t mla_last_launch_count(const mla_ctx* ctx) { return ctx ? ctx->last_launches : 0; }

mla_status mla_set_wait_limit(mla_ctx* ctx, uint64_t ns) {
  if (!ctx) return MLA_ERR_INVALID_ARG;
  ctx->gemm_wait_ns = ns;
  return MLA_OK;
}

size_t mla_mha_scratch_size(const mla_ctx* ctx, int32_t B, int32_t T, int32_t start_pos) {
  if (!ctx || B < 1 || T < 1 || start_pos < 0) return 0;
  return static_cast<size_t>(B) * (static_cast<size_t>(start_pos) + T) * ctx->cfg.n_heads *
         (kDn + kDv) * 2;
}

mla_status mla_prefill_chunk_mha(mla_ctx* ctx, const void* q_latent, void* residual,
                                 int32_t start_pos, int32_t T, const void* kv_cache,
                                 int64_t kv_stride_b, int64_t kv_stride_t, const void* pe_cache,
                                 int64_t pe_stride_b, int64_t pe_stride_t, int32_t B,
                                 void* kv_scratch, size_t scratch_bytes, void* out, float* lse,
                                 const void* wo, int32_t dim, void* y, cudaStream_t stream) {
  if (!ctx || !q_latent || !out || !kv_scratch) return MLA_ERR_INVALID_ARG;
  if (ctx->wq_scale) return MLA_ERR_UNSUPPORTED;   // bf16 weights only
  if (B < 1 || T < 1 || static_cast<int64_t>(B) * T > ctx->cfg.max_rows || start_pos < 0 ||
      static_cast<int64_t>(start_pos) + T > ctx->cfg.max_seq_len)
    return MLA_ERR_INVALID_ARG;
  if (scratch_bytes < mla_mha_scratch_size(ctx, B, T, start_pos)) return MLA_ERR_WORKSPACE;
  if (!aligned(q_latent, 16) || !aligned(out, 16) || !aligned(kv_scratch, 16) ||
      (residual && !aligned(residual, 16)) || (lse && !aligned(lse, 4)))
    return MLA_ERR_INVALID_ARG;
  if (wo && (!y || !aligned(wo, 16) || !aligned(y, 16) || dim < 8 || dim % 8 != 0 ||
             dim > 65536))
    return MLA_ERR_INVALID_ARG;
  if (!cache_args_ok(kv_cache, kv_stride_b, kv_stride_t, pe_cache, pe_stride_b, pe_stride_t))
    return MLA_ERR_INVALID_ARG;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev != ctx->device) return MLA_ERR_INVALID_ARG;
  return run_mha(ctx, q_latent, residual, start_pos, T, B, kv_cache, kv_stride_b, kv_stride_t,
                 pe_cache, pe_stride_b, pe_stride_t, kv_scratch, out, lse, wo, dim, y, stream);
}

mla_status mla_attach_producer(mla_ctx* ctx, int32_t dim, const void* wq_a, const void* wkv_a,
                               const float* kv_norm_gain) {
  if (!ctx || !wq_a || !wkv_a || !kv_norm_gain) return MLA_ERR_INVALID_ARG;
  if (dim < 64 || dim > 65536 || dim % 64 != 0) return MLA_ERR_UNSUPPORTED;
  if (!aligned(wq_a, 16) || !aligned(wkv_a, 16) || !aligned(kv_norm_gain, 16))
    return MLA_ERR_INVALID_ARG;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev != ctx->device) return MLA_ERR_INVALID_ARG;
  const uint64_t d = static_cast<uint64_t>(dim);
  CUtensorMap a, b;
  if (!make_map(&a, wq_a, d, kR, 1, d * 2, d * kR * 2, 64, 128, 1) ||
      !make_map(&b, wkv_a, d, kDk, 1, d * 2, d * kDk * 2, 64, 128, 1))
    return MLA_ERR_INVALID_ARG;
  ctx->tm_wqa = a;
  ctx->tm_wkva = b;
  ctx->kv_gain = kv_norm_gain;
  ctx->prod_dim = dim;
  return MLA_OK;
}

mla_status mla_produce(mla_ctx* ctx, const void* x, const int32_t* start_pos, int32_t start_pos_host,
                       int32_t T, int32_t B, void* kv_cache, int64_t kv_stride_b,
                       int64_t kv_stride_t, void* pe_cache, int64_t pe_stride_b,
                       int64_t pe_stride_t, void* q_latent, cudaStream_t stream) {
  if (!ctx || !x || !q_latent) return MLA_ERR_INVALID_ARG;
  if (ctx->prod_dim == 0) return MLA_ERR_INVALID_ARG;   // no producer weights attached
  if (B < 1 || T < 1 || static_cast<int64_t>(B) * T > ctx->cfg.max_rows) return MLA_ERR_INVALID_ARG;
  if (!start_pos && (start_pos_host < 0 ||
                     static_cast<int64_t>(start_pos_host) + T > ctx->cfg.max_seq_len))
    return MLA_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(q_latent, 16) || (start_pos && !aligned(start_pos, 4)))
    return MLA_ERR_INVALID_ARG;
  if (!cache_args_ok(kv_cache, kv_stride_b, kv_stride_t, pe_cache, pe_stride_b, pe_stride_t))
    return MLA_ERR_INVALID_ARG;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev != ctx->device) return MLA_ERR_INVALID_ARG;
  return run_produce(ctx, x, start_pos, start_pos_host, T, B, kv_cache, kv_stride_b, kv_stride_t,
                     pe_cache, pe_stride_b, pe_stride_t, q_latent, stream);
}

}  // extern "C"
