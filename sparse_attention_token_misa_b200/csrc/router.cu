// HISA block filter (block scores and candidate expansion) and the router's
// scratch layout.
//
// Block score of query t for key block j (all heads):
//     bs[t, j] = sum over h of w[t, h] * ReLU(q[t, h] . mean_j)
// HISA explainer (zhichai.net), section 三, Stage 1: the query is scored against
// the block representatives only and the top-m blocks are kept.  O(H * M * d)
// per query, a few percent of the token scoring; it runs on the fp32 CUDA cores
// with the query's heads and a chunk of block means staged in shared memory.
// (The MISA router, which reduces the same affinity over blocks instead of
// heads, runs on the tensor cores: route_tc.cu.)
#include "launch.h"
#include "misa_device.cuh"

namespace misa {

namespace {

constexpr int kThreads = 256;
constexpr int kChunk = 32;        // blocks per CTA (8 warps x 4 blocks)
constexpr int kPad = kD + 4;      // fp32 row pitch in shared memory (keeps float4 alignment, spreads banks)

// grid: (T, n_chunks).  Thread (warp jq, lane hp) owns heads hp + 32*a and
// blocks chunk*32 + 4*jq + u (u < 4); a warp reduces its heads per block.
__global__ void __launch_bounds__(kThreads)
block_score_kernel(const uint16_t* __restrict__ q, const float* __restrict__ w, const float* __restrict__ means,
                int64_t means_seq_stride, const int32_t* __restrict__ seq_of, const int32_t* __restrict__ prefix_len,
                int T, int H, int64_t L, int B, int M, int nseq_means,
                float* __restrict__ bscore,   // [T][bs_stride]
                int64_t bs_stride,
                uint32_t* __restrict__ err) {
  extern __shared__ float4 smem_f4[];
  float* sq = reinterpret_cast<float*>(smem_f4);   // [H][kPad]
  float* sm = sq + H * kPad;                        // [kChunk][kPad]
  __shared__ float sw[MISA_MAX_HEADS];

  const int t = blockIdx.x;
  const int chunk = blockIdx.y;
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int jq = tid >> 5;

  int seq = seq_of[t];
  if (seq < 0 || seq >= nseq_means) {
    if (tid == 0) record_error(err, MISA_DEVERR_BAD_SEQ);
    seq = 0;
  }
  // Visibility: a block is scored iff it lies wholly inside the query's prefix.
  const int64_t plen = prefix_len[t];

  // Stage q[t] (bf16 -> fp32), w[t] and the chunk's block means (zeros past
  // M).  Every global load of a thread is issued before any of them is used,
  // so the staging costs one memory latency, not one per loop trip.
  const uint16_t* qt = q + static_cast<int64_t>(t) * H * kD;
  const float* mb = means + static_cast<int64_t>(seq) * means_seq_stride;
  constexpr int kQPer = MISA_MAX_HEADS * (kD / 8) / kThreads;  // uint4 chunks of q per thread (max)
  constexpr int kMPer = kChunk * (kD / 4) / kThreads;           // float4 chunks of means per thread
  uint4 qv[kQPer];
  float4 mv[kMPer];
#pragma unroll
  for (int u = 0; u < kQPer; ++u) {
    const int i = tid + u * kThreads;
    qv[u] = i < H * (kD / 8) ? __ldg(reinterpret_cast<const uint4*>(qt) + i) : make_uint4(0u, 0u, 0u, 0u);
  }
#pragma unroll
  for (int u = 0; u < kMPer; ++u) {
    const int i = tid + u * kThreads;
    const int j = chunk * kChunk + i / (kD / 4);
    mv[u] = j < M ? __ldg(reinterpret_cast<const float4*>(mb + static_cast<int64_t>(j) * kD) + i % (kD / 4))
                  : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  const float wt = tid < H ? w[static_cast<int64_t>(t) * H + tid] : 0.f;
#pragma unroll
  for (int u = 0; u < kQPer; ++u) {
    const int i = tid + u * kThreads;
    if (i < H * (kD / 8)) {
      const int h = i / (kD / 8), c = i % (kD / 8);
      const __nv_bfloat162* pq = reinterpret_cast<const __nv_bfloat162*>(&qv[u]);
      float* dst = sq + h * kPad + c * 8;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 f = __bfloat1622float2(pq[k]);
        *reinterpret_cast<float2*>(dst + 2 * k) = f;
      }
    }
  }
#pragma unroll
  for (int u = 0; u < kMPer; ++u) {
    const int i = tid + u * kThreads;
    *reinterpret_cast<float4*>(sm + (i / (kD / 4)) * kPad + (i % (kD / 4)) * 4) = mv[u];
  }
  if (tid < H) sw[tid] = wt;
  __syncthreads();

  constexpr int kMaxHB = MISA_MAX_HEADS / 32;
  const int HB = (H + 31) / 32;
  float acc[kMaxHB][4];
#pragma unroll
  for (int a = 0; a < kMaxHB; ++a)
#pragma unroll
    for (int u = 0; u < 4; ++u) acc[a][u] = 0.f;

  const float* mrow = sm + (jq * 4) * kPad;
#pragma unroll 4
  for (int c = 0; c < kD; c += 4) {
    float4 mv[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) mv[u] = *reinterpret_cast<const float4*>(mrow + u * kPad + c);
#pragma unroll
    for (int a = 0; a < kMaxHB; ++a) {
      if (a < HB) {
        const int h = lane + 32 * a;
        const float4 qv = (h < H) ? *reinterpret_cast<const float4*>(sq + h * kPad + c) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          acc[a][u] = fmaf(qv.x, mv[u].x, acc[a][u]);
          acc[a][u] = fmaf(qv.y, mv[u].y, acc[a][u]);
          acc[a][u] = fmaf(qv.z, mv[u].z, acc[a][u]);
          acc[a][u] = fmaf(qv.w, mv[u].w, acc[a][u]);
        }
      }
    }
  }

  // A = w * ReLU(dot) on visible blocks, 0 elsewhere.
  bool vis[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int64_t j = static_cast<int64_t>(chunk) * kChunk + jq * 4 + u;
    const int64_t end = (j + 1) * B < L ? (j + 1) * B : L;
    vis[u] = (j < M) && (end <= plen);
  }
#pragma unroll
  for (int a = 0; a < kMaxHB; ++a) {
    const int h = lane + 32 * a;
    const float wh = (a < HB && h < H) ? sw[h] : 0.f;
#pragma unroll
    for (int u = 0; u < 4; ++u) acc[a][u] = vis[u] ? wh * fmaxf(acc[a][u], 0.f) : 0.f;
  }

    // HISA: block score = sum over heads (this thread's heads, then the warp).
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      float s = 0.f;
#pragma unroll
      for (int a = 0; a < kMaxHB; ++a) s += acc[a][u];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      const int j = chunk * kChunk + jq * 4 + u;
      // a block the prefix cuts (a causal query's own block) is always kept:
      // +inf; other blocks that are not wholly visible: -inf
      const int64_t jend = (static_cast<int64_t>(j) + 1) * B < L ? (static_cast<int64_t>(j) + 1) * B : L;
      const bool cut = static_cast<int64_t>(j) * B < plen && plen < jend;
      const float inf = __int_as_float(0x7f800000);
      if (lane == 0 && j < M) bscore[static_cast<int64_t>(t) * bs_stride + j] = vis[u] ? s : (cut ? inf : -inf);
  }
}

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

size_t affinity_smem_bytes(int H) { return static_cast<size_t>(H * kPad + kChunk * kPad) * sizeof(float); }

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

cudaError_t launch_hisa_block_scores(const uint16_t* q, const float* w, const float* means, int64_t means_seq_stride,
                                     const int32_t* seq_of, const int32_t* prefix_len, int T, int H, int64_t L, int B,
                                     int nseq_means, float* bscore, int64_t bs_stride, uint32_t* err,
                                     cudaStream_t stream) {
  const int M = static_cast<int>((L + B - 1) / B);
  const int nch = router_chunks(M);
  const size_t smem = affinity_smem_bytes(H);
  cudaError_t e = ensure_dynamic_smem(reinterpret_cast<const void*>(block_score_kernel), static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  block_score_kernel<<<dim3(T, nch), kThreads, smem, stream>>>(q, w, means, means_seq_stride, seq_of, prefix_len, T, H,
                                                               L, B, M, nseq_means, bscore, bs_stride, err);
  return cudaGetLastError();
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
