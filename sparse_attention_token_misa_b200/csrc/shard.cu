// Small kernels of the key-sharded (context-parallel) indexer: every rank
// holds keys [s0, s0 + L_shard) of every sequence, runs the router, the
// scoring and a local top-k over its shard, and the ranks exchange head
// importances (sum) and their local (score, token id) candidates.
//
// "MISA: Mixture of Indexer Sparse Attention for Long-Context LLM Inference"
// (gist.science), Methodology: the head importance is a sum over the visible
// blocks, so per-shard sums add up to it; the top-k of a union of per-shard
// top-k lists is the top-k of the whole row.
#include "launch.h"
#include "misa_device.cuh"

namespace misa {

namespace {

// out[t] = clamp(prefix_len[t] - s0, 0, L_shard): a key at local position s
// (global s0 + s) is visible iff s < out[t].
__global__ void shard_prefix_kernel(const int32_t* __restrict__ prefix_len, int T, int64_t s0, int64_t L_shard,
                                    int32_t* __restrict__ out) {
  pdl_wait_inputs();
  pdl_allow_next();
  for (int t = blockIdx.x * blockDim.x + threadIdx.x; t < T; t += gridDim.x * blockDim.x) {
    int64_t p = static_cast<int64_t>(prefix_len[t]) - s0;
    p = p < 0 ? 0 : (p > L_shard ? L_shard : p);
    out[t] = static_cast<int32_t>(p);
  }
}

// (score, global id) of each local pick; empty or out-of-range picks give
// (-inf, -1), which a later top-k never selects.
__global__ void gather_candidates_kernel(const float* __restrict__ scores, int T, int64_t n, int64_t row_stride,
                                         const int32_t* __restrict__ idx, int k, int64_t id_offset,
                                         float* __restrict__ out_scores, int32_t* __restrict__ out_ids) {
  pdl_wait_inputs();
  pdl_allow_next();
  const float kNegInf = -__int_as_float(0x7f800000);
  const int64_t total = static_cast<int64_t>(T) * k;
  for (int64_t x = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; x < total;
       x += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = x / k;
    const int32_t i = idx[x];
    const bool ok = i >= 0 && i < n;
    out_scores[x] = ok ? scores[t * row_stride + i] : kNegInf;
    out_ids[x] = ok ? static_cast<int32_t>(i + id_offset) : -1;
  }
}

}  // namespace

cudaError_t launch_shard_prefix(const int32_t* prefix_len, int T, int64_t s0, int64_t L_shard, int32_t* out,
                                cudaStream_t stream) {
  const int blocks = (T + 255) / 256;
  return launch_pdl(shard_prefix_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, stream, 0, prefix_len, T,
                    s0, L_shard, out);
}

cudaError_t launch_gather_candidates(const float* scores, int T, int64_t n, int64_t row_stride, const int32_t* idx,
                                     int k, int64_t id_offset, float* out_scores, int32_t* out_ids,
                                     cudaStream_t stream) {
  const int64_t total = static_cast<int64_t>(T) * k;
  const int sms = device_sm_count();
  if (sms <= 0) return cudaErrorInvalidDevice;
  int64_t blocks = (total + 255) / 256;
  if (blocks > static_cast<int64_t>(sms) * 8) blocks = static_cast<int64_t>(sms) * 8;
  return launch_pdl(gather_candidates_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, stream, 0, scores,
                    T, n, row_stride, idx, k, id_offset, out_scores, out_ids);
}

}  // namespace misa
