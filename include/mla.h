/*
 * mla.h — C ABI of the B200 (sm_100a) absorbed multi-head latent attention (MLA) library.
 *
 * The path, per query row (one new token of one sequence):
 *   a1  y  = RMSNorm(x (+ residual))                     fp32 math, bf16 out
 *   a2  q  = y · wq_bᵀ, viewed [H, nope+rope]             bf16 tensor cores, fp32 accumulate
 *   a3  q_pe = RoPE(q[..., nope:]) (interleaved pairs)    fused into the a2 epilogue
 *   a4  q_lat[h] = q_nope[h] · W_UK[h]                    (W_UK = first nope rows of wkv_b[h])
 *   a5  s[h, t] = (q_lat[h]·kv[t] + q_pe[h]·pe[t]) · softmax_scale
 *   a6  p = softmax_t(s)                                  fp32, online over key tiles
 *   a7  o_lat[h] = Σ_t p[h, t] · kv[t]
 *   a8  out[h] = W_UV[h] · o_lat[h]                       (W_UV = last v rows of wkv_b[h])
 *
 * Sources (page title · section):
 *   "DeepSeek-V3.2-Exp · Attention update": `rmsnorm` excerpt (a1, residual form) and `mla-decode`
 *     excerpt (the absorbed "MQA decode" branch: a4–a8);
 *   "DeepSeek-V3.2-Exp · Query heads": the six-step formula block, parameter table and the
 *     `mla-init` / `mla-queries` excerpts (a2, a3, softmax_scale = qk_head_dim^-0.5);
 *   "DeepSeek V4.1 · Query RMSNorm": RMSNorm formula (a1);
 *   "Kimi-K2 · value_states": W_UV shape and the non-absorbed form with its additive causal mask
 *     (prefill chunk semantics).
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller.  bf16 tensors are passed as
 *     `void*` and hold IEEE bfloat16 values; fp32 tensors as `float*`; positions as `int32_t*`.
 *   - Layouts are dense row-major in the order written; strides are in ELEMENTS.
 *   - Calls are asynchronous and ordered on `stream`; none synchronises the host.  Argument
 *     errors detected on the host return MLA_ERR_INVALID_ARG / MLA_ERR_UNSUPPORTED before anything
 *     is launched; a launch failure returns MLA_ERR_CUDA.  Problems only the device can see (a
 *     start position outside [0, max_seq_len), a bounded wait that gave up) are recorded in a
 *     device status word and reported by mla_sync_status().
 *   - Rows of every tensor handed to the tensor-memory-access (TMA) engine must start on a
 *     16-byte boundary: base pointers 16-byte aligned, row strides multiples of 8 elements.
 */
#ifndef MLA_B200_H
#define MLA_B200_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MLA_OK = 0,
    MLA_ERR_INVALID_ARG = 1,     /* null/misaligned pointer, size out of range, bad stride      */
    MLA_ERR_UNSUPPORTED = 2,     /* dimensions other than the ones the kernels are built for    */
    MLA_ERR_WORKSPACE = 3,       /* workspace missing, misaligned or smaller than required      */
    MLA_ERR_CUDA = 4,            /* a CUDA runtime/driver call or a kernel launch failed         */
    MLA_ERR_DEVICE_TIMEOUT = 5,  /* a kernel's bounded wait gave up (reported by mla_sync_status) */
    MLA_ERR_DEVICE_ARG = 6       /* a device-side argument (start position) was out of range    */
} mla_status;

/* Model dimensions ("Query heads" page, mla-init excerpt).  Supported: q_lora_rank = 1536,
 * kv_lora_rank = 512, qk_nope_head_dim = 128, qk_rope_head_dim = 64, v_head_dim = 128 and
 * n_heads a multiple of 16 in [16, 128]; anything else returns MLA_ERR_UNSUPPORTED. */
typedef struct {
    int32_t n_heads;            /* H                                                          */
    int32_t q_lora_rank;        /* R  = 1536                                                  */
    int32_t kv_lora_rank;       /* C  = 512                                                   */
    int32_t qk_nope_head_dim;   /* Dn = 128                                                   */
    int32_t qk_rope_head_dim;   /* Dr = 64                                                    */
    int32_t v_head_dim;         /* Dv = 128                                                   */
    float rope_theta;           /* RoPE base (10000)                                          */
    float softmax_scale;        /* 0 → (Dn+Dr)^-0.5                                           */
    float rms_eps;              /* q_norm epsilon (1e-6)                                      */
    int32_t max_rows;           /* largest B (decode) or B·T (prefill) a call may pass        */
    int32_t max_seq_len;        /* cache rows per sequence (>= 64); key indices < max_seq_len  */
} mla_config;

typedef struct mla_ctx mla_ctx; /* opaque; owns host metadata and views into the workspace   */

/* Human-readable name of a status code (static string). */
const char* mla_status_string(mla_status s);

/* Bytes of device workspace mla_init() needs for `cfg` (0 if cfg is invalid).  The workspace
 * holds the transposed W_UK copy, per-call intermediates (normalised latent, rotary table,
 * query heads, absorbed queries, attention partials, o_lat) and the device status word. */
size_t mla_workspace_size(const mla_config* cfg);

/* Create a context.
 *   q_norm_gain [R] fp32, wq_b [H·(Dn+Dr), R] bf16, wkv_b [H·(Dn+Dv), C] bf16 — nn.Linear
 *   layout [out, in]; per head, wq_b rows are Dn content rows then Dr rotary rows, and wkv_b rows
 *   are Dn W_UK rows then Dv W_UV rows ("Attention update" page, mla-decode excerpt).  Weights
 *   are BORROWED and must outlive the context.  `workspace` (device, 256-byte aligned, at least
 *   mla_workspace_size(cfg) bytes) is borrowed too.  One-time set-up kernels (W_UK transpose,
 *   zeroing) run on `stream`.  The context is bound to the current device.  On error *out is
 *   left NULL. */
mla_status mla_init(const mla_config* cfg, const float* q_norm_gain, const void* wq_b,
                    const void* wkv_b, void* workspace, size_t workspace_bytes,
                    cudaStream_t stream, mla_ctx** out);

/* mla_init with FP8 E4M3 block-scaled weights ("DeepSeek-V3.2-Exp · Attention update",
 * mla-decode: weight_dequant(wkv_b.weight, wkv_b.scale); the checkpoint stores FP8 weights with
 * one fp32 scale per 128 x 128 block).  The weights are dequantised inside the GEMMs, block by
 * block, to the bf16 values weight_dequant returns (code × scale, rounded to bf16), so the weight
 * bytes streamed per call are halved.
 *   wq_b_fp8 [H·(Dn+Dr), R] and wkv_b_fp8 [H·(Dn+Dv), C]: one E4M3 code per byte, same layouts
 *   as mla_init's bf16 weights; wq_b_scale [H·(Dn+Dr)/128, R/128] fp32 and wkv_b_scale
 *   [H·(Dn+Dv)/128, C/128] fp32: the scale of block (i/128, j/128).  Device pointers, borrowed.
 * Everything else (arguments, workspace, the calls that follow) as mla_init. */
mla_status mla_init_fp8(const mla_config* cfg, const float* q_norm_gain, const void* wq_b_fp8,
                        const float* wq_b_scale, const void* wkv_b_fp8, const float* wkv_b_scale,
                        void* workspace, size_t workspace_bytes, cudaStream_t stream,
                        mla_ctx** out);

void mla_destroy(mla_ctx* ctx);

/* a1 alone: y = RMSNorm(x (+ residual)) over rows of length `dim`.
 *   x [rows, dim] bf16; residual [rows, dim] bf16 or NULL — when given it is updated in place to
 *   x + residual (rounded to bf16) and the norm is taken of the fp32 sum ("Attention update"
 *   page, rmsnorm excerpt); gain [dim] fp32; y [rows, dim] bf16 (may not alias x).
 *   dim must be a multiple of 256 and at most 4096. */
mla_status mla_rmsnorm(const void* x, void* residual, const float* gain, int32_t rows,
                       int32_t dim, float eps, void* y, cudaStream_t stream);

/* Absorbed decode of one new token per sequence ("Attention update" page, mla-decode excerpt,
 * with the index mask keeping every key).
 *   q_latent [B, R] bf16 — the query latent before q_norm;
 *   residual [B, R] bf16 or NULL (in/out, see mla_rmsnorm);
 *   start_pos [B] int32 (device) — sequence b's new token has position start_pos[b], its latent is
 *     already in cache row start_pos[b], and it attends keys 0..start_pos[b];
 *   kv_cache — latent rows (C wide) of sequence b, key t at  kv_cache + b·kv_stride_b + t·kv_stride_t;
 *   pe_cache — rotated rotary-key rows (Dr wide), key t at  pe_cache + b·pe_stride_b + t·pe_stride_t.
 *     The pages keep two caches [B, max_seq_len, C] and [B, max_seq_len, Dr]; the packed layout
 *     [B, max_seq_len, C+Dr] is pe_cache = kv_cache + C with both strides (max_seq_len·(C+Dr),
 *     C+Dr).  Rows 0..max_seq_len-1 of every sequence must be addressable; rows past start_pos[b]
 *     never reach the result (their contents may be anything, NaN included);
 *   out [B, H, Dv] bf16;  lse [B, H] fp32 or NULL — natural-log sum of exp(scaled scores);
 *   logits [B, H, max_seq_len] fp32 or NULL — debug copy of the scaled scores s (only keys
 *     0..start_pos[b] are written).
 * 1 <= B <= cfg.max_rows.
 * Range: a row whose keys are split between SM pairs keeps each piece's normalised partial output
 * (a convex combination of cached latents) in fp16 before the log-sum-exp merge, so cached latent
 * values must lie within fp16's range (|value| <= 65504); larger values overflow to inf in those
 * rows only.  The same holds for mla_prefill_chunk. */
mla_status mla_decode(mla_ctx* ctx, const void* q_latent, void* residual, const int32_t* start_pos,
                      const void* kv_cache, int64_t kv_stride_b, int64_t kv_stride_t,
                      const void* pe_cache, int64_t pe_stride_b, int64_t pe_stride_t, int32_t B,
                      void* out, float* lse, float* logits, cudaStream_t stream);

/* Absorbed decode with the index mask of the V3.2 excerpt ("DeepSeek-V3.2-Exp · Attention
 * update", mla-decode: scores += full(-inf).scatter_(-1, topk_indices, 0); the selected keys come
 * from the caller, e.g. an indexer's top-k, "DeepSeek-V3.2-Exp · Indexer":
 * topk = min(index_topk, end_pos)).  Sequence b attends only keys topk_idx[b*k + j],
 * j < topk_len[b]; everything else is as mla_decode (the query's RoPE position is start_pos[b]).
 *   topk_idx [B, k] int32 (device): distinct key indices in [0, start_pos[b]] (a duplicate would
 *     count its key twice; an index outside [0, rows per sequence) is reported as
 *     MLA_ERR_DEVICE_ARG by mla_sync_status and read as key 0);
 *   topk_len [B] int32 (device): 1 <= topk_len[b] <= min(k, start_pos[b] + 1) (clamped into that
 *     range and reported as MLA_ERR_DEVICE_ARG otherwise).
 * The cache rows are gathered by index (four rows per TMA operation): kv_stride_b must be a whole
 * multiple of kv_stride_t, pe_stride_b of pe_stride_t, with the same quotient (rows per
 * sequence), as in the packed layout.  No logits output. */
mla_status mla_decode_sparse(mla_ctx* ctx, const void* q_latent, void* residual,
                             const int32_t* start_pos, const int32_t* topk_idx,
                             const int32_t* topk_len, int32_t k, const void* kv_cache,
                             int64_t kv_stride_b, int64_t kv_stride_t, const void* pe_cache,
                             int64_t pe_stride_b, int64_t pe_stride_t, int32_t B, void* out,
                             float* lse, cudaStream_t stream);

/* Absorbed attention for a chunk of T new tokens per sequence appended after `start_pos` cached
 * positions (causal: token t sees keys 0..start_pos+t, the additive -inf mask of the "Kimi-K2 ·
 * value_states" page's mla-prefill excerpt).  Cache rows start_pos..start_pos+T-1 must already
 * hold the chunk's own latents.  Cache arguments as for mla_decode.
 *   q_latent [B, T, R] bf16; residual [B, T, R] or NULL; out [B, T, H, Dv] bf16;
 *   lse [B, T, H] fp32 or NULL.  1 <= B·T <= cfg.max_rows, start_pos + T <= cfg.max_seq_len. */
mla_status mla_prefill_chunk(mla_ctx* ctx, const void* q_latent, void* residual, int32_t start_pos,
                             int32_t T, const void* kv_cache, int64_t kv_stride_b,
                             int64_t kv_stride_t, const void* pe_cache, int64_t pe_stride_b,
                             int64_t pe_stride_t, int32_t B, void* out, float* lse,
                             cudaStream_t stream);

/* The prefill chunk in the non-absorbed form ("Kimi-K2 · value_states", mla-prefill: every head's
 * key [W_UK kv ‖ k_pe] and value W_UV kv are rebuilt from the latent cache, then multi-head
 * attention with the additive causal mask and an fp32 softmax), followed optionally by the output
 * projection ("DeepSeek-V3.2-Exp · Attention update", mla-output: wo on the flattened heads).
 * Same result as mla_prefill_chunk up to rounding (the two forms are associative rewrites of
 * each other); this form does more arithmetic but no per-head absorption.
 *   Arguments as mla_prefill_chunk, plus:
 *   kv_scratch / scratch_bytes — device memory for the rebuilt keys and values of every head,
 *     at least mla_mha_scratch_size(ctx, B, T, start_pos) bytes (B·(start_pos+T)·H·256 bf16),
 *     16-byte aligned, owned by the caller (MLA_ERR_WORKSPACE if smaller);
 *   wo [dim, H·Dv] bf16 (nn.Linear layout) or NULL; dim a multiple of 8 in [8, 65536];
 *   y [B·T, dim] bf16 — wo applied to out (when wo is given).
 * Contexts made by mla_init_fp8 return MLA_ERR_UNSUPPORTED. */
size_t mla_mha_scratch_size(const mla_ctx* ctx, int32_t B, int32_t T, int32_t start_pos);
mla_status mla_prefill_chunk_mha(mla_ctx* ctx, const void* q_latent, void* residual,
                                 int32_t start_pos, int32_t T, const void* kv_cache,
                                 int64_t kv_stride_b, int64_t kv_stride_t, const void* pe_cache,
                                 int64_t pe_stride_b, int64_t pe_stride_t, int32_t B,
                                 void* kv_scratch, size_t scratch_bytes, void* out, float* lse,
                                 const void* wo, int32_t dim, void* y, cudaStream_t stream);

/* Latent attention without allocating memory (no counterpart on the source pages; an addition
 * for callers that cannot allocate device memory where they run, e.g. code confined to a
 * pre-reserved pool or given a fixed device budget by its host).
 *
 * Computes the attention step a5–a7 of mla_decode for caller-supplied absorbed queries:
 *   q_abs [rows, 128, C+Dr] bf16 — per row the absorbed query q_lat ‖ q_pe of each head, heads
 *     beyond n_heads padded with zeros (the layout mla_debug_copy(…, 2, …) returns);
 *   start_pos [rows] int32 (device) — row r attends keys 0..start_pos[r] of cache sequence r;
 *   caches and strides as for mla_decode, max_seq_len rows per sequence (>= 64);
 *   o_lat [rows, n_heads, C] bf16 — softmax-weighted sum of cached latents;
 *   lse [rows, n_heads] fp32 or NULL;
 *   status — device int32, required (NULL returns MLA_ERR_INVALID_ARG); the caller zeroes it
 *     before the call and reads it after synchronising; device-side problems are recorded there:
 *     6 (MLA_ERR_DEVICE_ARG) for a start position outside [0, max_seq_len), 5
 *     (MLA_ERR_DEVICE_TIMEOUT) for a bounded wait that gave up.
 * Argument checks are those of mla_decode (16-byte aligned rows and strides, strides below 2^40
 * bytes) plus 64 <= max_seq_len <= 2^24.
 * The library uses no memory but its inputs, its outputs and one fixed scratch array of about
 * 4.3 MB that every device loading the library holds until exit.  Limits: rows <= 4096 (more
 * returns MLA_ERR_INVALID_ARG); the split over keys uses at most 16 SM pairs.  The first call on
 * a device sets the array up (address lookup, kernel attribute), so make it before capturing a
 * stream into a graph.  All calls share the array: calls that can overlap on the GPU race and
 * must be serialised by the caller. */
mla_status mla_latent_attention_noalloc(const void* q_abs, const int32_t* start_pos,
                                        int32_t rows, int32_t n_heads, float softmax_scale,
                                        const void* kv_cache, int64_t kv_stride_b,
                                        int64_t kv_stride_t, const void* pe_cache,
                                        int64_t pe_stride_b, int64_t pe_stride_t,
                                        int32_t max_seq_len, void* o_lat, float* lse,
                                        int32_t* status, cudaStream_t stream);

/* Cache producer: the step upstream of the attention for new tokens ("DeepSeek-V3.2-Exp · Query
 * heads", mla-init: wq_a = Linear(dim, q_lora_rank), wkv_a = Linear(dim, kv_lora_rank +
 * qk_rope_head_dim), kv_norm = RMSNorm(kv_lora_rank); mla-queries: qr = q_norm(wq_a(x));
 * "Kimi-K2 · value_states", mla-init: the joint key-value down-projection also emits the shared
 * rotary key).  mla_attach_producer borrows the weights for later mla_produce calls:
 *   wq_a [R, dim] bf16, wkv_a [C + Dr, dim] bf16 (nn.Linear layout [out, in]; the first C outputs
 *   of wkv_a are the latent, the last Dr the rotary key), kv_norm_gain [C] fp32;
 *   dim a multiple of 64 in [64, 65536] (MLA_ERR_UNSUPPORTED otherwise).  Device pointers,
 *   16-byte aligned; they must outlive the context. */
mla_status mla_attach_producer(mla_ctx* ctx, int32_t dim, const void* wq_a, const void* wkv_a,
                               const float* kv_norm_gain);

/* For B sequences with T new tokens each (row r = b*T + t):
 *   q_latent[r] = x[r] wq_a^T  — [B*T, R] bf16 out, the input of mla_decode / mla_prefill_chunk;
 *   c = x[r] wkv_a^T (bf16); kv_cache row of (b, pos) = RMSNorm(c[:C]) with the kv_norm gain and
 *   the context's eps, bf16; pe_cache row of (b, pos) = interleaved RoPE of c[C:] at pos (the
 *   context's rope_theta), bf16 — with pos = start_pos[b] + t (start_pos: [B] int32 on the
 *   device) or start_pos_host + t when start_pos is NULL.  Cache arguments as for mla_decode;
 *   only the new rows are written.  x [B*T, dim] bf16.  1 <= B*T <= cfg.max_rows.  A position
 *   outside [0, max_seq_len) is not written and is reported as MLA_ERR_DEVICE_ARG by
 *   mla_sync_status.  The rows are written in stream order before any later mla_decode /
 *   mla_prefill_chunk on the same stream reads them (the pages write the cache, then attend). */
mla_status mla_produce(mla_ctx* ctx, const void* x, const int32_t* start_pos, int32_t start_pos_host,
                       int32_t T, int32_t B, void* kv_cache, int64_t kv_stride_b,
                       int64_t kv_stride_t, void* pe_cache, int64_t pe_stride_b,
                       int64_t pe_stride_t, void* q_latent, cudaStream_t stream);

/* Synchronise `stream`, then read and clear the device status word of `ctx`: MLA_OK,
 * MLA_ERR_DEVICE_TIMEOUT or MLA_ERR_DEVICE_ARG (or MLA_ERR_CUDA if the synchronisation failed). */
mla_status mla_sync_status(mla_ctx* ctx, cudaStream_t stream);

/* Stage timing.  When enabled, each decode / prefill call records CUDA events on its stream
 * around every kernel it launches.  mla_stage_times() waits for the last call's events and
 * writes up to `cap` per-kernel durations in milliseconds (kernel order of the call) and their
 * names; *n receives the number of stages. */
mla_status mla_enable_stage_timing(mla_ctx* ctx, int32_t enable);
mla_status mla_stage_times(mla_ctx* ctx, float* ms, const char** names, int32_t cap, int32_t* n);

/* Debug access to the last call's intermediates (device-to-device copy on `stream`).
 *   which: 0 = y [rows, R] bf16; 1 = q_nope [rows, H, Dn] bf16; 2 = absorbed query
 *   [rows, 128, C+Dr] bf16 (q_lat ‖ q_pe, heads padded to 128); 3 = o_lat [rows, H, C] bf16.
 *   `bytes` must not exceed the buffer (rows = the last call's row count). */
mla_status mla_debug_copy(mla_ctx* ctx, int32_t which, void* dst, size_t bytes,
                          cudaStream_t stream);

/* Test hook for the failure path: every wait inside the context's GEMM kernels (wq_b, the
 * absorption, W_UV, the producer's projections, the key/value rebuild, wo) gives up after `ns`
 * nanoseconds instead of 2 s (0 restores 2 s).  A wait that gives up makes the kernel record
 * MLA_ERR_DEVICE_TIMEOUT (read by mla_sync_status), drain its copies and MMAs, release its tensor
 * memory and return; the results of that call are then undefined, later calls are unaffected.
 * The attention kernels keep their 2 s bound. */
mla_status mla_set_wait_limit(mla_ctx* ctx, uint64_t ns);

/* Number of kernels the last decode / prefill / produce call launched. */
int32_t mla_last_launch_count(const mla_ctx* ctx);

#ifdef __cplusplus
}
#endif
#endif /* MLA_B200_H */
