// Pooled key blocks: the router's (and HISA's) block statistics, computed over
// a whole cache or kept up to date as keys are appended.
//
// "MISA: Mixture of Indexer Sparse Attention for Long-Context LLM Inference"
// (gist.science), Methodology: the prefix is split into M = ceil(L/B) blocks,
// each summarised by the mean of its indexer keys.  HISA explainer
// (zhichai.net), section 三, Stage 1: one mean-pooled representative per block;
// section 七 (潜在改进): overlapping blocks and max pooling as alternatives.
// Window j covers keys [j*S, min(j*S + B, L)), M = 1 + ceil(max(L - B, 0) / S)
// windows (S = B: the plain blocks); the statistic is the mean or the
// coordinate-wise maximum of the window's keys.
//
// One warp per (sequence, window).  A key row is 256 bytes = 16 lanes x 16 bytes,
// so a warp reads two rows per load (lanes 0-15 even rows, 16-31 odd rows),
// keeps 8 fp32 partial sums per lane and folds the two halves with one shuffle.
// Loads are 16-byte, coalesced, with several rows in flight per lane: the
// full-cache kernel is a single streaming pass over K and is HBM-bound.
//
// The append kernel writes the new keys into the cache and recomputes the
// blocks they touch (the open block's earlier keys are re-read) with the same
// summation order, so its means equal, bit for bit, those of a full recompute
// over the longer cache.
#include "launch.h"
#include "misa_device.cuh"

namespace misa {

namespace {

constexpr int kWarpsPerCta = 8;
constexpr int kUnroll = 4;  // row pairs in flight per lane

// Fold eight bf16 values into the running sums (kMax = false) or maxima.
template <bool kMax>
__device__ __forceinline__ void acc_bf16x8(float (&acc)[8], const uint4 v) {
  const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(p[i]);
    if (kMax) {
      acc[2 * i] = fmaxf(acc[2 * i], f.x);
      acc[2 * i + 1] = fmaxf(acc[2 * i + 1], f.y);
    } else {
      acc[2 * i] += f.x;
      acc[2 * i + 1] += f.y;
    }
  }
}

// Mean (or, with kMax, coordinate-wise maximum) of rows [s0, s1) of one
// window into out[0..128) and, when hi is not NULL, its split into two bf16
// rows: hi = bf16(stat), lo = bf16(stat - hi) (the tensor-core router's
// operands; a maximum of bf16 keys is a bf16 value, so its lo is 0);
// chunk_at(s) is the lane's 16-byte chunk of row s.  Every lane of the warp
// calls.
template <bool kMax, class ChunkAt>
__device__ __forceinline__ void block_pool_warp(int64_t s0, int64_t s1, ChunkAt chunk_at, float* out, uint16_t* hi,
                                                uint16_t* lo) {
  const int lane = threadIdx.x & 31;
  const int half = lane >> 4;   // which row of the pair
  const int chunk = lane & 15;  // 16-byte chunk of the row (8 bf16)
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = kMax ? -__int_as_float(0x7f800000) : 0.f;
  int64_t s = s0 + half;
  for (; s + 2 * (kUnroll - 1) < s1; s += 2 * kUnroll) {
    uint4 v[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) v[u] = chunk_at(s + 2 * u);
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) acc_bf16x8<kMax>(acc, v[u]);
  }
  for (; s < s1; s += 2) acc_bf16x8<kMax>(acc, chunk_at(s));
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float o = __shfl_xor_sync(0xffffffffu, acc[i], 16);
    acc[i] = kMax ? fmaxf(acc[i], o) : acc[i] + o;
  }
  if (half == 0) {
    const float inv = 1.0f / static_cast<float>(s1 - s0);
    float m[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) m[i] = kMax ? acc[i] : acc[i] * inv;
    float4* o = reinterpret_cast<float4*>(out + chunk * 8);
    o[0] = make_float4(m[0], m[1], m[2], m[3]);
    o[1] = make_float4(m[4], m[5], m[6], m[7]);
    if (hi) {
      uint32_t hw[4], lw[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const __nv_bfloat16 h0 = __float2bfloat16_rn(m[2 * c]);
        const __nv_bfloat16 h1 = __float2bfloat16_rn(m[2 * c + 1]);
        const __nv_bfloat16 l0 = __float2bfloat16_rn(m[2 * c] - __bfloat162float(h0));
        const __nv_bfloat16 l1 = __float2bfloat16_rn(m[2 * c + 1] - __bfloat162float(h1));
        hw[c] = static_cast<uint32_t>(__bfloat16_as_ushort(h0)) | (static_cast<uint32_t>(__bfloat16_as_ushort(h1)) << 16);
        lw[c] = static_cast<uint32_t>(__bfloat16_as_ushort(l0)) | (static_cast<uint32_t>(__bfloat16_as_ushort(l1)) << 16);
      }
      *reinterpret_cast<uint4*>(hi + chunk * 8) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
      *reinterpret_cast<uint4*>(lo + chunk * 8) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
    }
  }
}

template <bool kMax>
__global__ void __launch_bounds__(kWarpsPerCta * 32)
block_stats_kernel(const uint16_t* __restrict__ keys, int64_t nseq, int64_t L, int64_t key_seq_stride, int B, int S,
                   int64_t M, float* __restrict__ means, uint16_t* __restrict__ means_hi,
                   uint16_t* __restrict__ means_lo) {
  const int lane = threadIdx.x & 31;
  const int64_t gw = static_cast<int64_t>(blockIdx.x) * kWarpsPerCta + (threadIdx.x >> 5);
  if (gw >= nseq * M) return;
  const int64_t b = gw / M;
  const int64_t j = gw - b * M;
  const int64_t s0 = j * S;
  const int64_t s1 = (s0 + B < L) ? s0 + B : L;
  const uint16_t* base = keys + b * key_seq_stride + static_cast<int64_t>(lane & 15) * 8;
  const int64_t row = (b * M + j) * kD;
  block_pool_warp<kMax>(s0, s1, [&](int64_t s) { return __ldg(reinterpret_cast<const uint4*>(base + s * kD)); },
                        means + row, means_hi ? means_hi + row : nullptr, means_lo ? means_lo + row : nullptr);
}

// One warp per (sequence, touched window): copies its share of the new rows
// into the cache and recomputes the window's statistic from the cache's
// earlier rows and the new rows (read from new_keys, not from the cache being
// written).  The windows touched by the new rows [l0, l1) are those whose
// extent reaches past l0, from j_lo = (l0 < B ? 0 : (l0 - B) / S + 1) to the
// last window of the longer cache, M(l1) - 1; window j copies the new rows of
// [j*S, (j+1)*S) (the last one: up to l1), so every new row is copied once.
template <bool kMax>
__global__ void __launch_bounds__(kWarpsPerCta * 32)
append_keys_kernel(uint16_t* __restrict__ keys, int64_t nseq, int64_t key_seq_stride, int64_t L_cap,
                   const int32_t* __restrict__ len, const uint16_t* __restrict__ new_keys, int n_new, int B, int S,
                   int64_t blocks_per_seq, float* __restrict__ means, uint16_t* __restrict__ means_hi,
                   uint16_t* __restrict__ means_lo, int64_t means_seq_stride, uint32_t* __restrict__ err) {
  const int lane = threadIdx.x & 31;
  const int64_t gw = static_cast<int64_t>(blockIdx.x) * kWarpsPerCta + (threadIdx.x >> 5);
  if (gw >= nseq * blocks_per_seq) return;
  const int64_t b = gw / blocks_per_seq;
  const int64_t jj = gw - b * blocks_per_seq;
  const int64_t l0 = len[b];
  if (l0 < 0 || l0 + n_new > L_cap) {
    if (jj == 0 && lane == 0) record_error(err, MISA_DEVERR_BAD_LEN);
    return;
  }
  const int64_t l1 = l0 + n_new;
  const int64_t j_lo = l0 < B ? 0 : (l0 - B) / S + 1;
  const int64_t j_hi = (l1 > B ? (l1 - B + S - 1) / S : 0);  // last window of the longer cache
  const int64_t j = j_lo + jj;  // jj-th window touched by [l0, l1)
  if (j > j_hi) return;
  const int64_t s0 = j * S;
  const int64_t s1 = (s0 + B < l1) ? s0 + B : l1;
  const int64_t cofs = static_cast<int64_t>(lane & 15) * 8;
  uint16_t* cache = keys + b * key_seq_stride;
  const uint16_t* fresh = new_keys + b * static_cast<int64_t>(n_new) * kD;
  // this window's share of the new rows into the cache
  const int64_t c0 = s0 > l0 ? s0 : l0;
  const int64_t c1 = (j < j_hi && s0 + S < l1) ? s0 + S : l1;
  for (int64_t s = c0 + (lane >> 4); s < c1; s += 2)
    *reinterpret_cast<uint4*>(cache + s * kD + cofs) =
        __ldg(reinterpret_cast<const uint4*>(fresh + (s - l0) * kD + cofs));
  block_pool_warp<kMax>(
      s0, s1,
      [&](int64_t s) {
        return s < l0 ? __ldg(reinterpret_cast<const uint4*>(cache + s * kD + cofs))
                      : __ldg(reinterpret_cast<const uint4*>(fresh + (s - l0) * kD + cofs));
      },
      means + b * means_seq_stride + j * kD, means_hi ? means_hi + b * means_seq_stride + j * kD : nullptr,
      means_lo ? means_lo + b * means_seq_stride + j * kD : nullptr);
}

}  // namespace

int64_t num_windows(int64_t L, int64_t B, int64_t S) { return 1 + (L > B ? (L - B + S - 1) / S : 0); }

cudaError_t launch_block_stats(const uint16_t* keys, int64_t nseq, int64_t L, int64_t key_seq_stride, int B, int S,
                               bool pool_max, float* means, uint16_t* means_hi, uint16_t* means_lo,
                               cudaStream_t stream) {
  const int64_t M = num_windows(L, B, S);
  const int64_t warps = nseq * M;
  const int64_t ctas = (warps + kWarpsPerCta - 1) / kWarpsPerCta;
  if (ctas > 0x7fffffff) return cudaErrorInvalidValue;
  auto kern = pool_max ? block_stats_kernel<true> : block_stats_kernel<false>;
  kern<<<static_cast<unsigned>(ctas), kWarpsPerCta * 32, 0, stream>>>(keys, nseq, L, key_seq_stride, B, S, M, means,
                                                                     means_hi, means_lo);
  return cudaGetLastError();
}

cudaError_t launch_append_keys(uint16_t* keys, int64_t nseq, int64_t key_seq_stride, int64_t L_cap,
                               const int32_t* len, const uint16_t* new_keys, int n_new, int B, int S, bool pool_max,
                               float* means, uint16_t* means_hi, uint16_t* means_lo, int64_t means_seq_stride,
                               uint32_t* err, cudaStream_t stream) {
  // [l0, l0 + n_new) touches at most floor((n_new - 1 + B) / S) + 1 windows
  // (ceil(n_new / B) + 1 blocks when S = B)
  const int64_t blocks_per_seq = (static_cast<int64_t>(n_new) - 1 + B) / S + 1;
  const int64_t warps = nseq * blocks_per_seq;
  const int64_t ctas = (warps + kWarpsPerCta - 1) / kWarpsPerCta;
  if (ctas > 0x7fffffff) return cudaErrorInvalidValue;
  auto kern = pool_max ? append_keys_kernel<true> : append_keys_kernel<false>;
  kern<<<static_cast<unsigned>(ctas), kWarpsPerCta * 32, 0, stream>>>(keys, nseq, key_seq_stride, L_cap, len,
                                                                     new_keys, n_new, B, S, blocks_per_seq, means,
                                                                     means_hi, means_lo, means_seq_stride, err);
  return cudaGetLastError();
}

}  // namespace misa
