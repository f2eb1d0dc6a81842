// k_rmsnorm.cu — a1: q_norm RMSNorm with optional fused residual add.
//
// "DeepSeek-V3.2-Exp · Attention update", rmsnorm excerpt: in fp32, u = x (+ residual); the new
// residual is u cast back to the input type; y = gain * u * rsqrt(mean(u^2) + eps), cast back.
// "DeepSeek V4.1 · Query RMSNorm" gives the same formula.
//
// One warp per row; each lane holds dim/32 values in registers (16-byte bf16 vector loads and
// stores, fully coalesced), the sum of squares is reduced with warp shuffles.  The decode/prefill
// chain also uses this kernel to emit two small side outputs so that no extra launch is needed:
//   * the rotary table (cos, sin) of each row's position for the 32 interleaved pairs
//     ("Query heads" page: R [T positions, 32 pairs]), angles evaluated in double precision;
//   * the cumulative key count of the rows (block 0), used by the attention and combine kernels
//     to split the flattened key range evenly across SM pairs.
#include "internal.h"
#include "tc100.cuh"

namespace mla {

__device__ __forceinline__ int row_position(const RmsParams& p, int row, bool* bad) {
  int pos;
  if (p.start_pos_dev) {
    pos = p.start_pos_dev[row];
  } else {
    pos = p.start_pos + row % p.T;
  }
  if (pos < 0 || pos >= p.max_seq_len) {
    *bad = true;
    pos = pos < 0 ? 0 : p.max_seq_len - 1;
  }
  return pos;
}

// Keys a row attends: every key 0..position (dense), or the row's count of selected keys
// (index-mask decode), clamped to [1, min(K, position + 1)] with the clamp reported.
__device__ __forceinline__ int row_keys(const RmsParams& p, int row, bool* bad) {
  const int pos = row_position(p, row, bad);
  if (!p.topk_len) return pos + 1;
  int n = p.topk_len[row];
  const int cap = pos + 1 < p.topk_k ? pos + 1 : p.topk_k;
  if (n < 1 || n > cap) {
    *bad = true;
    n = n < 1 ? 1 : cap;
  }
  return n;
}

__device__ void key_prefix_block(const RmsParams& p) {
  // 128 threads; thread t owns rows [t*chunk, (t+1)*chunk).  Block-wide scan of the per-thread
  // key counts (warp shuffles, then the four warp totals), then each thread writes its rows'
  // prefix and assigns the attention pairs whose first key falls in one of its rows.
  __shared__ long long warp_total[4];
  const int t = threadIdx.x, lane = t & 31, w = t >> 5;
  const int chunk = (p.rows + 127) / 128;
  const int r0 = min(p.rows, t * chunk), r1 = min(p.rows, r0 + chunk);
  long long local = 0;
  bool bad = false;
  for (int r = r0; r < r1; ++r) local += row_keys(p, r, &bad);
  long long incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  if (lane == 31) warp_total[w] = incl;
  __syncthreads();
  long long acc = incl - local, total = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const long long v = warp_total[i];
    if (i < w) acc += v;
    total += v;
  }
  if (t == 0) p.row_prefix[0] = 0;
  // pair q begins at key floor(total * q / pairs): it starts in row r iff that key lies in
  // [prefix[r], prefix[r+1]), i.e. q in [ceil(prefix[r] * pairs / total), ceil(prefix[r+1] * ...))
  const int pairs = p.pair_row ? active_pairs(total, p.n_pairs, p.min_keys_per_pair) : 0;
  auto first_pair_at = [&](long long key) -> long long {
    return (key * pairs + total - 1) / total;
  };
  for (int r = r0; r < r1; ++r) {
    const long long R0 = acc;
    acc += row_keys(p, r, &bad);
    p.row_prefix[r + 1] = acc;
    if (p.pair_row) {
      const long long qa = first_pair_at(R0), qb = first_pair_at(acc);
      const long long q1 = qb < pairs ? qb : pairs;
      for (long long q = qa; q < q1; ++q) p.pair_row[q] = r;
      if (p.row_pieces) {
        // pair qa begins at or after R0; it begins exactly there iff total*qa < (R0+1)*pairs.
        // Otherwise the row's first key belongs to pair qa-1, which began in an earlier row.
        const bool starts_here = qa < pairs && total * qa < (R0 + 1) * pairs;
        const int plo = static_cast<int>(starts_here ? qa : qa - 1);
        const int phi = static_cast<int>(q1 - 1);
        p.row_pieces[r] = make_int2(2 * plo + (starts_here ? 0 : 1), phi);
      }
    }
  }
  if (bad) atomicCAS(p.status, kDevOk, kDevBadArg);
}

template <int NCH>
__global__ void __launch_bounds__(128) rmsnorm_kernel(const RmsParams p) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * 4 + warp;
  const bool live = row < p.rows;
  // The row's loads go out first, so that block 0's key prefix (its own round trip to memory)
  // overlaps them instead of preceding them.  The gain is preloaded too when it fits.
  constexpr bool kPreGain = NCH <= 8;
  uint4 xv[NCH], rv[NCH];
  float4 gv[kPreGain ? 2 * NCH : 1];
  const uint4* xr = reinterpret_cast<const uint4*>(p.x + static_cast<size_t>(row) * p.dim);
  uint4* rr = p.residual ? reinterpret_cast<uint4*>(p.residual + static_cast<size_t>(row) * p.dim)
                         : nullptr;
  const float4* g4 = reinterpret_cast<const float4*>(p.gamma);
  if (live) {
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
      const int idx = lane + 32 * c;
      xv[c] = xr[idx];
      if (rr) rv[c] = rr[idx];
      if constexpr (kPreGain) {
        gv[2 * c] = g4[2 * idx];
        gv[2 * c + 1] = g4[2 * idx + 1];
      }
    }
  }
  // The kernels after this one start early (programmatic dependent launch) and the attention
  // kernel reads the key prefix before it waits for its predecessors: block 0 therefore writes
  // the prefix first and makes it visible before any block lets the next kernel start.
  if (blockIdx.x == 0 && p.row_prefix) {
    key_prefix_block(p);
    __threadfence();
    __syncthreads();
  }
  pdl_launch_dependents();
  if (live) {
    float u[NCH][8];
    float ss = 0.f;
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
      const int idx = lane + 32 * c;
      const __nv_bfloat16* xb = reinterpret_cast<const __nv_bfloat16*>(&xv[c]);
#pragma unroll
      for (int i = 0; i < 8; ++i) u[c][i] = __bfloat162float(xb[i]);
      if (rr) {
        const __nv_bfloat16* rb = reinterpret_cast<const __nv_bfloat16*>(&rv[c]);
        uint4 ov;
        uint32_t* o32 = reinterpret_cast<uint32_t*>(&ov);
#pragma unroll
        for (int i = 0; i < 8; ++i) u[c][i] += __bfloat162float(rb[i]);
#pragma unroll
        for (int i = 0; i < 4; ++i) o32[i] = pack_bf16x2(u[c][2 * i], u[c][2 * i + 1]);
        rr[idx] = ov;
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) ss = fmaf(u[c][i], u[c][i], ss);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float inv = rsqrtf(ss / static_cast<float>(p.dim) + p.eps);
    uint4* yr = reinterpret_cast<uint4*>(p.y + static_cast<size_t>(row) * p.dim);
#pragma unroll
    for (int c = 0; c < NCH; ++c) {
      const int idx = lane + 32 * c;
      float4 ga, gb;
      if constexpr (kPreGain) {
        ga = gv[2 * c];
        gb = gv[2 * c + 1];
      } else {
        ga = g4[2 * idx];
        gb = g4[2 * idx + 1];
      }
      const float g[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
      uint4 ov;
      uint32_t* o32 = reinterpret_cast<uint32_t*>(&ov);
#pragma unroll
      for (int i = 0; i < 4; ++i)
        o32[i] = pack_bf16x2(g[2 * i] * (u[c][2 * i] * inv), g[2 * i + 1] * (u[c][2 * i + 1] * inv));
      yr[idx] = ov;
    }
    if (p.rope_tab) {
      bool bad = false;
      const int pos = row_position(p, row, &bad);
      // theta_i = theta^(-2i/64); lane i owns pair i
      const double inv_freq = exp(-2.0 * static_cast<double>(lane) / kDr * p.rope_log_theta);
      double sn, cs;
      sincos(static_cast<double>(pos) * inv_freq, &sn, &cs);
      p.rope_tab[static_cast<size_t>(row) * kRopePairs + lane] =
          make_float2(static_cast<float>(cs), static_cast<float>(sn));
    }
  }
}

cudaError_t launch_rmsnorm(const RmsParams& p, cudaStream_t s) {
  const int nch = p.dim / 256;
  dim3 grid((p.rows + 3) / 4), block(128);
  switch (nch) {
#define MLA_RMS_CASE(n) \
  case n:               \
    rmsnorm_kernel<n><<<grid, block, 0, s>>>(p); \
    break;
    MLA_RMS_CASE(1) MLA_RMS_CASE(2) MLA_RMS_CASE(3) MLA_RMS_CASE(4) MLA_RMS_CASE(5)
    MLA_RMS_CASE(6) MLA_RMS_CASE(7) MLA_RMS_CASE(8) MLA_RMS_CASE(9) MLA_RMS_CASE(10)
    MLA_RMS_CASE(11) MLA_RMS_CASE(12) MLA_RMS_CASE(13) MLA_RMS_CASE(14) MLA_RMS_CASE(15)
    MLA_RMS_CASE(16)
#undef MLA_RMS_CASE
    default:
      return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

// ------------------------------------------------------------------------------------------
// Cache producer, second half: the wkv_a output c = [latent (512) ‖ rotary key (64)] of each new
// token → kv_cache row = RMSNorm(latent) with the kv_norm gain, pe_cache row = RoPE(key) at the
// token's position ("Query heads" mla-init: kv_norm = RMSNorm(kv_lora_rank); "Kimi-K2 ·
// value_states" mla-init: the joint down-projection also emits the shared rotary key).
// One warp per row: lane l holds latent columns 16l .. 16l+15 and rotary pair l.
// ------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(128) kv_finish_kernel(const KvFinishParams p) {
  pdl_launch_dependents();
  pdl_wait();   // c comes from the wkv_a GEMM
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * 4 + warp;
  if (row >= p.rows) return;
  const int b = row / p.T, t = row - b * p.T;
  const long long pos = static_cast<long long>(p.start_pos_dev ? p.start_pos_dev[b] : p.start_pos) + t;
  if (pos < 0 || pos >= p.max_seq_len) {   // recorded, nothing written
    if (lane == 0) atomicCAS(p.status, kDevOk, kDevBadArg);
    return;
  }
  const bf16* c = p.c + static_cast<size_t>(row) * kDk;
  const uint4* c4 = reinterpret_cast<const uint4*>(c);
  const uint4 a0 = c4[2 * lane], a1 = c4[2 * lane + 1];
  const __nv_bfloat162 kp = reinterpret_cast<const __nv_bfloat162*>(c + kC)[lane];
  const float4* g4 = reinterpret_cast<const float4*>(p.gain) + 4 * lane;
  const float4 ga = g4[0], gb = g4[1], gc = g4[2], gd = g4[3];
  float u[16];
  const __nv_bfloat16* ab = reinterpret_cast<const __nv_bfloat16*>(&a0);
  const __nv_bfloat16* bb = reinterpret_cast<const __nv_bfloat16*>(&a1);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    u[i] = __bfloat162float(ab[i]);
    u[8 + i] = __bfloat162float(bb[i]);
  }
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) ss = fmaf(u[i], u[i], ss);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float inv = rsqrtf(ss / static_cast<float>(kC) + p.eps);
  const float g[16] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w,
                       gc.x, gc.y, gc.z, gc.w, gd.x, gd.y, gd.z, gd.w};
  uint32_t o[8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
    o[i] = pack_bf16x2(g[2 * i] * (u[2 * i] * inv), g[2 * i + 1] * (u[2 * i + 1] * inv));
  uint4* kv = reinterpret_cast<uint4*>(p.kv_cache + b * p.kv_sb + pos * p.kv_st) + 2 * lane;
  kv[0] = make_uint4(o[0], o[1], o[2], o[3]);
  kv[1] = make_uint4(o[4], o[5], o[6], o[7]);
  // rotary key: pair `lane` rotated by pos * theta^(-2 lane / 64), angle in double precision
  const double inv_freq = exp(-2.0 * static_cast<double>(lane) / kDr * p.rope_log_theta);
  double sn, cs;
  sincos(static_cast<double>(pos) * inv_freq, &sn, &cs);
  const float x0 = __low2float(kp), x1 = __high2float(kp);
  const float fc = static_cast<float>(cs), fs = static_cast<float>(sn);
  reinterpret_cast<uint32_t*>(p.pe_cache + b * p.pe_sb + pos * p.pe_st)[lane] =
      pack_bf16x2(x0 * fc - x1 * fs, x0 * fs + x1 * fc);
}

cudaError_t launch_kv_finish(const KvFinishParams& p, cudaStream_t s, bool pdl) {
  LaunchCfg lc(dim3((p.rows + 3) / 4), dim3(128), 0, s, pdl);
  return cudaLaunchKernelEx(&lc.cfg, kv_finish_kernel, p);
}

// Cumulative key counts of decode rows only (one block); used by the no-allocation attention
// entry point, which has no RMSNorm launch to carry it.
__global__ void __launch_bounds__(128) key_prefix_kernel(const RmsParams p) { key_prefix_block(p); }

cudaError_t launch_key_prefix(const RmsParams& p, cudaStream_t s) {
  key_prefix_kernel<<<1, 128, 0, s>>>(p);
  return cudaGetLastError();
}

}  // namespace mla
