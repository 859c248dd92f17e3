// HISA candidate expansion and the router's scratch layout.
//
// HISA explainer (zhichai.net), section 三, Stage 2: the tokens of the top-m
// blocks are the candidates the full indexer scores.  (The block scores of
// Stage 1 are computed on the tensor cores by the router's kernel:
// route_tc.cu.)
#include "launch.h"
#include "misa_device.cuh"

namespace misa {

namespace {

constexpr int kChunk = 32;        // blocks per partial-importance chunk of the router's scratch

// cand[t][i*B + r] = blocks[t][i]*B + r if the slot is filled and the id is
// inside the prefix (and the cache), else -1.
__global__ void hisa_expand_kernel(const int32_t* __restrict__ blocks, const int32_t* __restrict__ prefix_len,
                                   int T, int m, int B, int64_t L, int32_t* __restrict__ cand) {
  const int64_t n = static_cast<int64_t>(m) * B;
  const int t = blockIdx.x;
  const int64_t limit = prefix_len[t] < L ? prefix_len[t] : L;
  for (int64_t p = static_cast<int64_t>(blockIdx.y) * blockDim.x + threadIdx.x; p < n;
       p += static_cast<int64_t>(gridDim.y) * blockDim.x) {
    const int i = static_cast<int>(p / B);
    const int r = static_cast<int>(p - static_cast<int64_t>(i) * B);
    const int32_t blk = blocks[static_cast<int64_t>(t) * m + i];
    int64_t id = -1;
    if (blk >= 0) {
      id = static_cast<int64_t>(blk) * B + r;
      if (id >= limit) id = -1;
    }
    cand[static_cast<int64_t>(t) * n + p] = static_cast<int32_t>(id);
  }
}

}  // namespace

int router_chunks(int M) { return (M + kChunk - 1) / kChunk; }

size_t router_counters_offset(int T, int H, int64_t L, int B) {
  const int64_t M = (L + B - 1) / B;
  const size_t part = static_cast<size_t>(T) * router_chunks(static_cast<int>(M)) * H * sizeof(float);
  return (part + 255) / 256 * 256;
}

size_t router_scratch_bytes(int T, int H, int64_t L, int B, int q_block) {
  const int G = (T + q_block - 1) / q_block;
  return router_counters_offset(T, H, L, B) + static_cast<size_t>(G) * sizeof(unsigned);
}

cudaError_t launch_hisa_expand(const int32_t* blocks, const int32_t* prefix_len, int T, int m, int B, int64_t L,
                               int32_t* cand, cudaStream_t stream) {
  const int64_t n = static_cast<int64_t>(m) * B;
  const int threads = 256;
  int64_t gx = (n + threads - 1) / threads;
  if (gx > 1024) gx = 1024;
  hisa_expand_kernel<<<dim3(T, static_cast<unsigned>(gx)), threads, 0, stream>>>(blocks, prefix_len, T, m, B, L, cand);
  return cudaGetLastError();
}

}  // namespace misa
