// Mean-pooled key blocks: the router's (and HISA's) block statistics.
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
// kernel is a single streaming pass over K and is HBM-bound.
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

__global__ void __launch_bounds__(kWarpsPerCta * 32)
block_stats_kernel(const uint16_t* __restrict__ keys, int64_t nseq, int64_t L, int64_t key_seq_stride, int B,
                   int64_t M, float* __restrict__ means) {
  const int lane = threadIdx.x & 31;
  const int64_t gw = static_cast<int64_t>(blockIdx.x) * kWarpsPerCta + (threadIdx.x >> 5);
  if (gw >= nseq * M) return;
  const int64_t b = gw / M;
  const int64_t j = gw - b * M;
  const int64_t s0 = j * B;
  const int64_t s1 = (s0 + B < L) ? s0 + B : L;
  const int half = lane >> 4;   // which row of the pair
  const int chunk = lane & 15;  // 16-byte chunk of the row (8 bf16)
  const uint16_t* base = keys + b * key_seq_stride + static_cast<int64_t>(chunk) * 8;

  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;

  int64_t s = s0 + half;
  for (; s + 2 * (kUnroll - 1) < s1; s += 2 * kUnroll) {
    uint4 v[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u)
      v[u] = __ldg(reinterpret_cast<const uint4*>(base + (s + 2 * u) * kD));
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) acc_bf16x8(acc, v[u]);
  }
  for (; s < s1; s += 2) acc_bf16x8(acc, __ldg(reinterpret_cast<const uint4*>(base + s * kD)));

#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], 16);

  if (half == 0) {
    const float inv = 1.0f / static_cast<float>(s1 - s0);
    float4* out = reinterpret_cast<float4*>(means + (b * M + j) * kD + chunk * 8);
    out[0] = make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
    out[1] = make_float4(acc[4] * inv, acc[5] * inv, acc[6] * inv, acc[7] * inv);
  }
}

}  // namespace

cudaError_t launch_block_stats(const uint16_t* keys, int64_t nseq, int64_t L, int64_t key_seq_stride, int B,
                               float* means, cudaStream_t stream) {
  const int64_t M = (L + B - 1) / B;
  const int64_t warps = nseq * M;
  const int64_t ctas = (warps + kWarpsPerCta - 1) / kWarpsPerCta;
  if (ctas > 0x7fffffff) return cudaErrorInvalidValue;
  block_stats_kernel<<<static_cast<unsigned>(ctas), kWarpsPerCta * 32, 0, stream>>>(keys, nseq, L, key_seq_stride,
                                                                                   B, M, means);
  return cudaGetLastError();
}

}  // namespace misa
