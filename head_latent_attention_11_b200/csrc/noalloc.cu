// noalloc.cu — latent attention entry point that allocates no memory.
//
// Some callers cannot allocate device memory at the point where they run attention: code that
// runs inside a pre-reserved memory pool it must not grow, plug-ins handed a fixed device budget
// by their host, or a process whose allocator is owned by another framework.  This entry point
// serves them: the caller passes its inputs and outputs, and the only other device memory used
// is the fixed scratch array below, part of the library's image on every device that loads it.
//
// The scratch holds the per-row key prefix, the first row of each SM pair's key range, the
// per-row piece records and the split-K partial outputs of at most kNoAllocPairs SM pairs; the
// caller's status word receives device-side errors.  Limits: rows <= kNoAllocMaxRows; the attention
// splits over at most kNoAllocPairs pairs (fewer SMs than the context path on large GPUs).
//
// Set-up: the first call on a device (with that device current) resolves the array's device
// address with cudaGetSymbolAddress and sets the attention kernel's shared-memory attribute;
// make that first call before capturing the stream into a CUDA graph.  Every call shares the
// same array, so calls that may overlap on the GPU (different streams, different threads)
// race on it and must be serialised by the caller.
#include <math.h>

#include <mutex>

#include "mla.h"
#include "internal.h"
#include "tc100.cuh"

namespace mla {
namespace {

constexpr int kNoAllocMaxRows = 4096;
constexpr int kNoAllocPairs = 16;
constexpr size_t kOffPrefix = 0;
constexpr size_t kOffPartO = kOffPrefix + ((static_cast<size_t>(kNoAllocMaxRows) + 1) * 8 + 255) / 256 * 256;
constexpr size_t kOffPartLse = kOffPartO + static_cast<size_t>(kNoAllocPairs) * 2 * 128 * kC * 2;
constexpr size_t kOffPairRow = kOffPartLse + static_cast<size_t>(kNoAllocPairs) * 2 * 128 * 4;
constexpr size_t kOffRowPieces = kOffPairRow + 256;
constexpr size_t kScratchBytes = kOffRowPieces + static_cast<size_t>(kNoAllocMaxRows) * 8;

// ~4.3 MB on every device that loads the library, kept until the process exits.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

struct DeviceSetup {
  bool done = false;
  unsigned char* scratch = nullptr;   // device address of g_noalloc_scratch on that device
};
DeviceSetup g_setup[64];
std::mutex g_setup_mu;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace mla

using namespace mla;

extern "C" mla_status mla_latent_attention_noalloc(
    const void* q_abs, const int32_t* start_pos, int32_t rows, int32_t n_heads,
    float softmax_scale, const void* kv_cache, int64_t kv_stride_b, int64_t kv_stride_t,
    const void* pe_cache, int64_t pe_stride_b, int64_t pe_stride_t, int32_t max_seq_len,
    void* o_lat, float* lse, int32_t* status, cudaStream_t stream) {
  if (!q_abs || !start_pos || !o_lat || !status) return MLA_ERR_INVALID_ARG;
  if (rows < 1 || rows > kNoAllocMaxRows) return MLA_ERR_INVALID_ARG;   // beyond the scratch
  if (n_heads < 16 || n_heads > 128 || n_heads % 16 != 0) return MLA_ERR_UNSUPPORTED;
  if (max_seq_len < 64 || max_seq_len > (1 << 24) || !(softmax_scale > 0.f) ||
      !isfinite(softmax_scale))
    return MLA_ERR_INVALID_ARG;
  if (!aligned16(q_abs) || !aligned16(o_lat) || (reinterpret_cast<uintptr_t>(start_pos) & 3u) ||
      (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) ||
      (reinterpret_cast<uintptr_t>(status) & 3u))
    return MLA_ERR_INVALID_ARG;
  if (!cache_args_ok(kv_cache, kv_stride_b, kv_stride_t, pe_cache, pe_stride_b, pe_stride_t))
    return MLA_ERR_INVALID_ARG;

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return MLA_ERR_CUDA;
  unsigned char* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_setup_mu);
    DeviceSetup& su = g_setup[dev];
    if (!su.done) {
      void* ptr = nullptr;
      if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) return MLA_ERR_CUDA;
      if (attention_prepare() != cudaSuccess) return MLA_ERR_CUDA;
      su.scratch = static_cast<unsigned char*>(ptr);
      su.done = true;
    }
    scratch = su.scratch;
  }
  int* st = status;
  long long* prefix = reinterpret_cast<long long*>(scratch + kOffPrefix);
  __half* part_o = reinterpret_cast<__half*>(scratch + kOffPartO);
  float* part_lse = reinterpret_cast<float*>(scratch + kOffPartLse);
  int* pair_row = reinterpret_cast<int*>(scratch + kOffPairRow);
  int2* row_pieces = reinterpret_cast<int2*>(scratch + kOffRowPieces);

  const int pairs = attention_pairs() < kNoAllocPairs ? attention_pairs() : kNoAllocPairs;
  AttnMaps am;
  if (!make_attention_maps(&am, kv_cache, kv_stride_b, kv_stride_t, pe_cache, pe_stride_b,
                           pe_stride_t, rows, max_seq_len, q_abs, rows, o_lat, n_heads, part_o, pairs))
    return MLA_ERR_INVALID_ARG;

  // the prefix and partials in the scratch array are written before they are read within the
  // call; nothing in it needs clearing
  RmsParams rp{};
  rp.rows = rows;
  rp.T = 1;
  rp.start_pos_dev = start_pos;
  rp.max_seq_len = max_seq_len;
  rp.row_prefix = prefix;
  rp.pair_row = pair_row;
  rp.row_pieces = row_pieces;
  rp.n_pairs = pairs;
  rp.min_keys_per_pair = kMinKeysPerPair;
  rp.status = st;
  if (launch_key_prefix(rp, stream) != cudaSuccess) return MLA_ERR_CUDA;

  AttnParams ap{};
  ap.row_prefix = prefix;
  ap.qabs = static_cast<const bf16*>(q_abs);
  ap.rows = rows;
  ap.T = 1;
  ap.n_heads = n_heads;
  ap.scale = softmax_scale;
  ap.scale_log2 = softmax_scale * 1.4426950408889634f;
  ap.min_keys_per_pair = kMinKeysPerPair;
  ap.o_lat = static_cast<bf16*>(o_lat);
  ap.lse_out = lse;
  ap.max_seq_len = max_seq_len;
  ap.part_o = part_o;
  ap.part_lse = part_lse;
  ap.pair_row = pair_row;
  ap.status = st;
  if (launch_attention(am, ap, pairs, stream, false) != cudaSuccess) return MLA_ERR_CUDA;

  CombineParams cp{};
  cp.row_prefix = prefix;
  cp.rows = rows;
  cp.n_heads = n_heads;
  cp.n_pairs = pairs;
  cp.min_keys_per_pair = kMinKeysPerPair;
  cp.part_o = part_o;
  cp.part_lse = part_lse;
  cp.row_pieces = row_pieces;
  cp.o_lat = static_cast<bf16*>(o_lat);
  cp.lse_out = lse;
  cp.status = st;
  if (launch_combine(cp, stream, false) != cudaSuccess) return MLA_ERR_CUDA;
  return MLA_OK;
}
