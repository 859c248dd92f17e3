// Mean-pooled key blocks: the router's (and HISA's) block statistics, computed
// over a whole cache or kept up to date as keys are appended.
//
// "MISA: Mixture of Indexer Sparse Attention for Long-Context LLM Inference"
// (gist.science), Methodology: the prefix is split into M = ceil(L/B) blocks,
// each summarised by the mean of its indexer keys.  HISA explainer
// (zhichai.net), section 三, Stage 1: one mean-pooled representative per block.
//
// One warp per (sequence, block).  A key row is 256 bytes = 16 lanes x 16 bytes,
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

__device__ __forceinline__ void acc_bf16x8(float (&acc)[8], const uint4 v) {
  const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(p[i]);
    acc[2 * i] += f.x;
    acc[2 * i + 1] += f.y;
  }
}

// Mean of rows [s0, s1) of one block into out[0..128) and, when hi is not
// NULL, its split into two bf16 rows: hi = bf16(mean), lo = bf16(mean - hi)
// (the tensor-core router's operands); chunk_at(s) is the lane's 16-byte chunk
// of row s.  Every lane of the warp calls.
template <class ChunkAt>
__device__ __forceinline__ void block_mean_warp(int64_t s0, int64_t s1, ChunkAt chunk_at, float* out, uint16_t* hi,
                                                uint16_t* lo) {
  const int lane = threadIdx.x & 31;
  const int half = lane >> 4;   // which row of the pair
  const int chunk = lane & 15;  // 16-byte chunk of the row (8 bf16)
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;
  int64_t s = s0 + half;
  for (; s + 2 * (kUnroll - 1) < s1; s += 2 * kUnroll) {
    uint4 v[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) v[u] = chunk_at(s + 2 * u);
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) acc_bf16x8(acc, v[u]);
  }
  for (; s < s1; s += 2) acc_bf16x8(acc, chunk_at(s));
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], 16);
  if (half == 0) {
    const float inv = 1.0f / static_cast<float>(s1 - s0);
    float m[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) m[i] = acc[i] * inv;
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

__global__ void __launch_bounds__(kWarpsPerCta * 32)
block_stats_kernel(const uint16_t* __restrict__ keys, int64_t nseq, int64_t L, int64_t key_seq_stride, int B,
                   int64_t M, float* __restrict__ means, uint16_t* __restrict__ means_hi,
                   uint16_t* __restrict__ means_lo) {
  const int lane = threadIdx.x & 31;
  const int64_t gw = static_cast<int64_t>(blockIdx.x) * kWarpsPerCta + (threadIdx.x >> 5);
  if (gw >= nseq * M) return;
  const int64_t b = gw / M;
  const int64_t j = gw - b * M;
  const int64_t s0 = j * B;
  const int64_t s1 = (s0 + B < L) ? s0 + B : L;
  const uint16_t* base = keys + b * key_seq_stride + static_cast<int64_t>(lane & 15) * 8;
  const int64_t row = (b * M + j) * kD;
  block_mean_warp(s0, s1, [&](int64_t s) { return __ldg(reinterpret_cast<const uint4*>(base + s * kD)); },
                  means + row, means_hi ? means_hi + row : nullptr, means_lo ? means_lo + row : nullptr);
}

// One warp per (sequence, touched block): copies the new rows of its block
// into the cache and recomputes the block's mean from the cache's earlier
// rows and the new rows (read from new_keys, not from the cache being
// written).
__global__ void __launch_bounds__(kWarpsPerCta * 32)
append_keys_kernel(uint16_t* __restrict__ keys, int64_t nseq, int64_t key_seq_stride, int64_t L_cap,
                   const int32_t* __restrict__ len, const uint16_t* __restrict__ new_keys, int n_new, int B,
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
  const int64_t j = l0 / B + jj;  // jj-th block touched by [l0, l1)
  const int64_t s0 = j * B;
  if (s0 >= l1) return;
  const int64_t s1 = (s0 + B < l1) ? s0 + B : l1;
  const int64_t cofs = static_cast<int64_t>(lane & 15) * 8;
  uint16_t* cache = keys + b * key_seq_stride;
  const uint16_t* fresh = new_keys + b * static_cast<int64_t>(n_new) * kD;
  // the new rows of this block into the cache
  for (int64_t s = (s0 > l0 ? s0 : l0) + (lane >> 4); s < s1; s += 2)
    *reinterpret_cast<uint4*>(cache + s * kD + cofs) =
        __ldg(reinterpret_cast<const uint4*>(fresh + (s - l0) * kD + cofs));
  block_mean_warp(
      s0, s1,
      [&](int64_t s) {
        return s < l0 ? __ldg(reinterpret_cast<const uint4*>(cache + s * kD + cofs))
                      : __ldg(reinterpret_cast<const uint4*>(fresh + (s - l0) * kD + cofs));
      },
      means + b * means_seq_stride + j * kD, means_hi ? means_hi + b * means_seq_stride + j * kD : nullptr,
      means_lo ? means_lo + b * means_seq_stride + j * kD : nullptr);
}

}  // namespace

cudaError_t launch_block_stats(const uint16_t* keys, int64_t nseq, int64_t L, int64_t key_seq_stride, int B,
                               float* means, uint16_t* means_hi, uint16_t* means_lo, cudaStream_t stream) {
  const int64_t M = (L + B - 1) / B;
  const int64_t warps = nseq * M;
  const int64_t ctas = (warps + kWarpsPerCta - 1) / kWarpsPerCta;
  if (ctas > 0x7fffffff) return cudaErrorInvalidValue;
  block_stats_kernel<<<static_cast<unsigned>(ctas), kWarpsPerCta * 32, 0, stream>>>(keys, nseq, L, key_seq_stride,
                                                                                   B, M, means, means_hi, means_lo);
  return cudaGetLastError();
}

cudaError_t launch_append_keys(uint16_t* keys, int64_t nseq, int64_t key_seq_stride, int64_t L_cap,
                               const int32_t* len, const uint16_t* new_keys, int n_new, int B, float* means,
                               uint16_t* means_hi, uint16_t* means_lo, int64_t means_seq_stride, uint32_t* err,
                               cudaStream_t stream) {
  // [l0, l0 + n_new) touches at most ceil(n_new / B) + 1 blocks
  const int64_t blocks_per_seq = (n_new + B - 1) / B + 1;
  const int64_t warps = nseq * blocks_per_seq;
  const int64_t ctas = (warps + kWarpsPerCta - 1) / kWarpsPerCta;
  if (ctas > 0x7fffffff) return cudaErrorInvalidValue;
  append_keys_kernel<<<static_cast<unsigned>(ctas), kWarpsPerCta * 32, 0, stream>>>(
      keys, nseq, key_seq_stride, L_cap, len, new_keys, n_new, B, blocks_per_seq, means, means_hi, means_lo,
      means_seq_stride, err);
  return cudaGetLastError();
}

}  // namespace misa
