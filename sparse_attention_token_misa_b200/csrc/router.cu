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

// cand[t][i*B + r] = blocks[t][i]*S + r (window i of the ascending choice,
// windows S tokens apart) if the slot is filled, the id is inside the prefix
// (and the cache) and no earlier chosen window lists it already, else -1.
// The chosen windows ascend, so the earlier windows' last token is the
// previous window's: id is new iff id >= blocks[t][i-1]*S + B.  With S = B the
// windows do not overlap and the last test never fires.
__global__ void hisa_expand_kernel(const int32_t* __restrict__ blocks, const int32_t* __restrict__ prefix_len,
                                   int T, int m, int B, int S, int64_t L, int32_t* __restrict__ cand) {
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
      id = static_cast<int64_t>(blk) * S + r;
      const int32_t prev = i > 0 ? blocks[static_cast<int64_t>(t) * m + i - 1] : -1;
      if (id >= limit || (prev >= 0 && id < static_cast<int64_t>(prev) * S + B)) id = -1;
    }
    cand[static_cast<int64_t>(t) * n + p] = static_cast<int32_t>(id);
  }
}

}  // namespace

int router_chunks(int M) { return (M + kChunk - 1) / kChunk; }

size_t router_counters_offset_m(int T, int H, int64_t M) {
  const size_t part = static_cast<size_t>(T) * router_chunks(static_cast<int>(M)) * H * sizeof(float);
  return (part + 255) / 256 * 256;
}

size_t router_scratch_bytes_m(int T, int H, int64_t M, int q_block) {
  const int G = (T + q_block - 1) / q_block;
  return router_counters_offset_m(T, H, M) + static_cast<size_t>(G) * sizeof(unsigned);
}

size_t router_counters_offset(int T, int H, int64_t L, int B) { return router_counters_offset_m(T, H, (L + B - 1) / B); }

size_t router_scratch_bytes(int T, int H, int64_t L, int B, int q_block) {
  return router_scratch_bytes_m(T, H, (L + B - 1) / B, q_block);
}

cudaError_t launch_hisa_expand(const int32_t* blocks, const int32_t* prefix_len, int T, int m, int B, int S,
                               int64_t L, int32_t* cand, cudaStream_t stream) {
  const int64_t n = static_cast<int64_t>(m) * B;
  const int threads = 256;
  int64_t gx = (n + threads - 1) / threads;
  if (gx > 1024) gx = 1024;
  hisa_expand_kernel<<<dim3(T, static_cast<unsigned>(gx)), threads, 0, stream>>>(blocks, prefix_len, T, m, B, S, L,
                                                                                 cand);
  return cudaGetLastError();
}

}  // namespace misa
