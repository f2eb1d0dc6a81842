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

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

struct Layout {
  size_t status, w_ukt, y, rope, q_nope, qabs, o_lat, part_o, part_lse, prefix, pair_row,
      row_pieces, total;
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

#define MLA_TRY(expr)                               \
  do {                                              \
    cudaError_t _e = (expr);                        \
    if (_e != cudaSuccess) return MLA_ERR_CUDA;     \
  } while (0)

// The whole path for `rows` query rows.  decode: start_pos_dev != null, T = 1.
mla_status run_path(mla_ctx* c, const void* q_latent, void* residual, const int32_t* start_pos_dev,
                    int start_pos, int T, int B, const void* kv, int64_t kv_sb, int64_t kv_st,
                    const void* pe, int64_t pe_sb, int64_t pe_st, void* out, float* lse,
                    float* logits, cudaStream_t s) {
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
                           rows, c->o_lat(), H, c->part_o(), c->n_pairs))
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
  clk.mark("wq_b_rope");
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
  clk.mark("absorb_w_uk");
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
  MLA_TRY(launch_gemm(c->tm_wuv, tm_olat, g3, H, s, true));
  ++launches;
  clk.finish();

  c->last_rows = rows;
  c->last_launches = launches;
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

mla_status mla_init(const mla_config* cfg, const float* q_norm_gain, const void* wq_b,
                    const void* wkv_b, void* workspace, size_t workspace_bytes, cudaStream_t stream,
                    mla_ctx** out) {
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
    if (gemm_prepare() != cudaSuccess || attention_prepare() != cudaSuccess) return MLA_ERR_CUDA;
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
  for (int i = 0; i <= kMaxStages; ++i) c->ev[i] = nullptr;

  const int H = cfg->n_heads;
  bool ok = make_map(&c->tm_wq, c->wq_b, kR, static_cast<uint64_t>(H) * kDq, 1, kR * 2,
                     static_cast<uint64_t>(H) * kDq * kR * 2, 64, 128, 1) &&
            make_map(&c->tm_wukt, c->w_ukt(), kDn, kC, H, kDn * 2,
                     static_cast<uint64_t>(kC) * kDn * 2, 64, 128, 1) &&
            make_map(&c->tm_wuv, c->wkv_b, kC, kDn + kDv, H, kC * 2,
                     static_cast<uint64_t>(kDn + kDv) * kC * 2, 64, 128, 1);
  if (!ok) {
    delete c;
    return MLA_ERR_CUDA;
  }
  if (cudaMemsetAsync(workspace, 0, L.total, stream) != cudaSuccess ||
      launch_transpose_uk(c->wkv_b, c->w_ukt(), H, stream) != cudaSuccess) {
    delete c;
    return MLA_ERR_CUDA;
  }
  *out = c;
  return MLA_OK;
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

}  // extern "C"
