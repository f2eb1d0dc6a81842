// internal.h — parameter blocks shared between the host launch code (api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace mla {

typedef __nv_bfloat16 bf16;

// Fixed model dimensions the kernels are built for ("Query heads" page, mla-init excerpt).
constexpr int kR = 1536;     // q_lora_rank
constexpr int kC = 512;      // kv_lora_rank
constexpr int kDn = 128;     // qk_nope_head_dim
constexpr int kDr = 64;      // qk_rope_head_dim
constexpr int kDv = 128;     // v_head_dim
constexpr int kDq = kDn + kDr;        // 192 query features per head
constexpr int kDk = kC + kDr;         // 576-wide absorbed query / cache row
constexpr int kHPad = 128;            // heads padded to one 128-row MMA tile
constexpr int kRopePairs = kDr / 2;   // 32
constexpr int kAttnKeysPerTile = 32;  // cache rows per attention tile (TMA box height)

// ---------------------------------------------------------------------------------------
// a1: RMSNorm (+ residual) with the rotary table and the per-row key prefix as side outputs
// ---------------------------------------------------------------------------------------
struct RmsParams {
  const bf16* x;            // [rows, dim]
  bf16* residual;           // [rows, dim] or null (in/out)
  const float* gamma;       // [dim]
  bf16* y;                  // [rows, dim]
  int rows;
  int dim;
  float eps;
  // rotary table (cos, sin) per row and pair; null to skip
  float2* rope_tab;         // [rows, 32]
  double rope_log_theta;    // ln(theta)
  // positions: decode → start_pos_dev[row]; prefill → start_pos + row % T
  const int32_t* start_pos_dev;
  int start_pos;
  int T;
  int max_seq_len;
  // key prefix over rows (written by block 0); null to skip
  long long* row_prefix;    // [rows + 1]
  // first row of each attention pair's key range (written by block 0 after the prefix);
  // null to skip.  n_pairs / min_keys_per_pair as given to the attention kernel.
  int* pair_row;            // [n_pairs]
  // per row: the first and last pair its keys fall in, {2 * plo + (plo began in an earlier
  // row), phi} (written with pair_row; null to skip)
  int2* row_pieces;         // [rows]
  int n_pairs;
  int min_keys_per_pair;
  int* status;
  // index-mask decode: per-row count of selected keys (null: dense) and the list capacity K
  const int32_t* topk_len;
  int topk_k;
};

// ---------------------------------------------------------------------------------------
// Cache producer: kv_norm + key RoPE of the wkv_a output, written to the caller's cache rows
// ---------------------------------------------------------------------------------------
struct KvFinishParams {
  const bf16* c;            // [rows, 576]: wkv_a output (latent ‖ rotary key), bf16
  const float* gain;        // [512] kv_norm gain
  bf16* kv_cache;           // row of key t of sequence b at kv_cache + b*kv_sb + t*kv_st
  long long kv_sb, kv_st;
  bf16* pe_cache;
  long long pe_sb, pe_st;
  int rows, T;              // row = b*T + t
  const int32_t* start_pos_dev;   // [B] or null (then start_pos for every sequence)
  int start_pos;
  int max_seq_len;
  float eps;
  double rope_log_theta;
  int* status;
};

// ---------------------------------------------------------------------------------------
// a2/a4/a8: bf16 tensor-core GEMM  D[m, n] = sum_k A[g][m, k] * B[g][n, k]  (both K-major)
// ---------------------------------------------------------------------------------------
enum EpiKind : int {
  kEpiStore = 0,   // out0[n*ld_n0 + g*ld_g0 + m] = bf16(D)
  kEpiWqbRope = 1, // wq_b: nope rows → q_nope, rope rows → rotated → absorbed-query buffer
};

struct GemmParams {
  int M, N, K;
  int a_row_off;           // row offset of the A tile inside its tensor map
  int epi;
  bf16* out0;
  long long ld_n0, ld_g0;
  bf16* out1;              // kEpiWqbRope: absorbed-query buffer [rows, 128, 576]
  const float2* rope_tab;  // [N, 32]
  int n_heads;
  int* status;
  // W_UV only, N <= 64 (merge mode): B = o_lat is built in shared memory by the epilogue warps,
  // merging the attention's split-K pieces of each token (row) for the CTA's head; uncut rows
  // are read from o_lat, merged rows are written back to o_lat (and lse_out when given).
  int bmerge;
  const long long* row_prefix;  // [rows + 1]
  const __half* part_o;         // [pairs, 2, 128, 512]
  const float* part_lse;        // [pairs, 2, 128]
  const int2* row_pieces;       // [rows] see RmsParams::row_pieces
  bf16* o_lat;                  // [rows, n_heads, 512]
  float* lse_out;               // [rows, n_heads] or null
  int n_pairs, min_keys_per_pair;
  // FP8 E4M3 weights (null: bf16 A): A holds fp8 codes; the value of A[g][m][k] is its code times
  // a_scale[g * a_sg + ((m + a_row_off) / 128) * a_sm + (k / 128) * a_sk] (128 x 128 blocks)
  const float* a_scale;
  long long a_sg, a_sm, a_sk;
  long long a_scale_n;     // elements of a_scale (an index at or past it is reported, not read)
  int b_g0;                // B is shared by every batch g (its batch coordinate is 0)
  unsigned long long wait_limit_ns;   // bound of every wait in the kernel (0: the 2 s default)
};

// ---------------------------------------------------------------------------------------
// Non-absorbed prefill: multi-head attention over keys / values rebuilt from the latent
// ---------------------------------------------------------------------------------------
struct FmhaParams {
  bf16* out;              // [B*T, H, 128]
  float* lse;             // [B*T, H] or null
  int T, B, n_heads, start_pos;
  float scale_log2;
  int* status;
  unsigned long long wait_limit_ns;
};
struct FmhaMaps {
  CUtensorMap qn;         // q_nope {128, H, rows},           box {64, 1, 128}
  CUtensorMap qp;         // absorbed query {576, 128, rows}, box {64, 1, 128} (q_pe at 512)
  CUtensorMap kvb;        // rebuilt keys / values {H*256, keys, B}, box {64, 128, 1}
  CUtensorMap pe;         // rotary cache {64, L, B},          box {64, 128, 1}
};
cudaError_t fmha_prepare();
cudaError_t launch_fmha(const FmhaMaps& m, const FmhaParams& p, cudaStream_t s, bool pdl);

// ---------------------------------------------------------------------------------------
// a5–a7: latent flash attention (cluster of two CTAs splits the 576-wide contraction and the
// 512-wide value dimension), split over keys; rows are query tokens, heads are the MMA M dim.
// ---------------------------------------------------------------------------------------
struct AttnParams {
  const long long* row_prefix;  // [rows + 1] cumulative key counts
  const bf16* qabs;             // [rows, 128, 576] absorbed query (q_lat ‖ q_pe), heads padded
  int rows;
  int T;                        // prefill tokens per sequence (decode: 1)
  int n_heads;
  float scale_log2;             // softmax_scale * log2(e)
  float scale;                  // softmax_scale
  int min_keys_per_pair;
  bf16* o_lat;                  // [rows, H, 512] bf16 (rows attended by one pair only)
  float* lse_out;               // [rows, H] or null
  float* logits;                // [B, H, max_seq_len] or null (decode debug)
  int max_seq_len;
  __half* part_o;               // [pairs, 2, 128, 512] fp16 normalised partial outputs
  float* part_lse;              // [pairs, 2, 128]
  const int* pair_row;          // [pairs] first row of each pair's key range, or null
  int* status;
  unsigned long long wait_limit_ns;   // bound of every wait in the kernel (0: the 2 s default)
  // index-mask decode (null: dense): key j of row r is cache row topk_idx[r * topk_k + j] of its
  // sequence, gathered through the 2-D maps kv2 / pe2 (row = b * seq_rows + index)
  const int32_t* topk_idx;
  int topk_k;
  long long seq_rows;           // cache rows per sequence in the 2-D view (batch stride / row stride)
};

struct CombineParams {
  const long long* row_prefix;
  int rows;
  int n_heads;
  int n_pairs;                  // pairs the attention kernel launched
  int min_keys_per_pair;
  const __half* part_o;
  const float* part_lse;
  const int2* row_pieces;       // [rows] see RmsParams::row_pieces
  bf16* o_lat;
  float* lse_out;
  int* status;
};

// cuTensorMapEncodeTiled through the runtime's driver entry point (no interleave, L2 256-byte
// promotion, zero fill).  dims/box have `rank` entries, strides (bytes) rank - 1.
bool encode_tiled(CUtensorMap* m, CUtensorMapDataType dt, int rank, const void* base,
                  const uint64_t* dims, const uint64_t* strides, const uint32_t* box,
                  CUtensorMapSwizzle swizzle);

// Launch configuration; with pdl set the kernel is launched with programmatic stream
// serialisation: its CTAs may start while the previous kernel of the stream is still running, and
// it waits (griddepcontrol.wait) before it reads or writes anything that kernel touches.
struct LaunchCfg {
  cudaLaunchConfig_t cfg;
  cudaLaunchAttribute attr[1];
  LaunchCfg(dim3 grid, dim3 block, size_t smem, cudaStream_t s, bool pdl) {
    cfg = cudaLaunchConfig_t{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
  }
};

// Launchers (defined next to their kernels).  pdl: see LaunchCfg.
cudaError_t launch_rmsnorm(const RmsParams& p, cudaStream_t s);
cudaError_t launch_key_prefix(const RmsParams& p, cudaStream_t s);   // row_prefix only
cudaError_t launch_kv_finish(const KvFinishParams& p, cudaStream_t s, bool pdl);
cudaError_t launch_gemm(const CUtensorMap& ta, const CUtensorMap& tb, const GemmParams& p,
                        int batches, cudaStream_t s, bool pdl);
// Tensor maps of the attention kernel, built on the host for each call (all 128-byte swizzle).
struct AttnMaps {
  CUtensorMap kv;    // latent cache  bf16 {512, max_seq_len, batch}, box {64, 32, 1}
  CUtensorMap pe;    // rotary cache  bf16 {64, max_seq_len, batch},  box {32, 32, 1}, 64-B swizzle
  CUtensorMap q;     // absorbed queries bf16 {576, 128, rows},       box {64, 128, 1}
  CUtensorMap qpe;   // the same, 64-byte swizzle,                     box {32, 128, 1}
  CUtensorMap o;     // o_lat         bf16 {512, n_heads, rows},      box {64, 32, 1}
  CUtensorMap part;  // split partials fp16 {512, pairs * 2 * 128},   box {64, 32}
  // index-mask decode only: the caches as 2-D row arrays for tile::gather4 (one-row boxes)
  CUtensorMap kv2;   // bf16 {512, batch * seq_rows}, box {64, 1}
  CUtensorMap pe2;   // bf16 {64, batch * seq_rows},  box {32, 1}, 64-B swizzle
};
// Strides in elements; false if a map cannot be encoded (alignment, sizes).
bool make_attention_maps(AttnMaps* m, const void* kv, int64_t kv_sb, int64_t kv_st, const void* pe,
                         int64_t pe_sb, int64_t pe_st, int batch, int max_seq_len, const void* qabs,
                         int rows, const void* o_lat, int n_heads, const void* part_o, int pairs);
// The 2-D gather maps (kv2, pe2) for the index-mask decode; needs batch strides that are whole
// multiples of the row strides.
bool make_gather_maps(AttnMaps* m, const void* kv, int64_t kv_sb, int64_t kv_st, const void* pe,
                      int64_t pe_sb, int64_t pe_st, int batch);
cudaError_t launch_attention(const AttnMaps& m, const AttnParams& p, int n_pairs, cudaStream_t s,
                             bool pdl);
cudaError_t launch_combine(const CombineParams& p, cudaStream_t s, bool pdl);
cudaError_t launch_transpose_uk(const bf16* wkv_b, bf16* w_ukt, int n_heads, cudaStream_t s);
cudaError_t launch_transpose_uk_fp8(const uint8_t* wkv_b, uint8_t* w_ukt, int n_heads,
                                    cudaStream_t s);
cudaError_t gemm_prepare();        // one-time per-device attribute set-up
cudaError_t attention_prepare();

// Smallest key range the attention kernel gives one SM pair (split-K granularity).
constexpr int kMinKeysPerPair = 256;

// Host-side check of the cache arguments shared by every entry point that reads the cache:
// non-null, 16-byte aligned bases, rows at least C (kv) / Dr (pe) wide, row and batch strides
// multiples of 16 bytes and below 2^40 bytes (tensor-map limits).  Strides in elements.
inline bool cache_args_ok(const void* kv, int64_t kv_sb, int64_t kv_st, const void* pe,
                          int64_t pe_sb, int64_t pe_st) {
  auto al16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  if (!kv || !pe || !al16(kv) || !al16(pe)) return false;
  if (kv_st < kC || pe_st < kDr || kv_sb < 1 || pe_sb < 1) return false;
  if ((kv_st * 2) % 16 || (pe_st * 2) % 16 || (kv_sb * 2) % 16 || (pe_sb * 2) % 16) return false;
  if (kv_st * 2 >= (1ll << 40) || pe_st * 2 >= (1ll << 40) || kv_sb * 2 >= (1ll << 40) ||
      pe_sb * 2 >= (1ll << 40))
    return false;
  return true;
}

// Token-tile width the GEMM launcher picks for N token rows (the B operand's TMA box height).
inline int gemm_bn(int n) { return n <= 32 ? 32 : n <= 64 ? 64 : n <= 128 ? 128 : 256; }

// Number of cluster pairs the attention kernel uses on this device (SMs / 2).
int attention_pairs();

// Pair partition of the flattened key range, shared by the attention and combine kernels.
__host__ __device__ inline int active_pairs(long long total_keys, int launched, int min_keys) {
  long long want = (total_keys + min_keys - 1) / min_keys;
  if (want < 1) want = 1;
  return want < launched ? static_cast<int>(want) : launched;
}
__host__ __device__ inline long long pair_begin(long long total_keys, int pairs, int p) {
  return total_keys * p / pairs;
}

// Row containing flattened key e: largest r with prefix[r] <= e (plain loads: the prefix may
// have been written earlier by the calling kernel).
__device__ __forceinline__ int row_of_key(const long long* prefix, int rows, long long e) {
  int lo = 0, hi = rows - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (prefix[mid] <= e) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

}  // namespace mla
