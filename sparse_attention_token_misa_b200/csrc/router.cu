// Block-level affinity shared by the MISA router and the HISA block filter,
// the router's per-query-block head selection, and HISA's candidate expansion.
//
// Affinity of head h of query t with key block j:
//     A[t, h, j] = w[t, h] * ReLU(q[t, h] . mean_j)
// "MISA: Mixture of Indexer Sparse Attention for Long-Context LLM Inference"
// (gist.science), Methodology: per-head affinities against block-aggregated
// keys, aggregated into a head importance, top-h heads kept (cost O(H_I * M)).
// HISA explainer (zhichai.net), section 三, Stage 1: the query is scored against
// the block representatives only, top-m blocks kept.
//
// The router reduces A over blocks (and over the queries of a routing
// decision; the last CTA of a decision to finish, found with an atomic
// counter, sums the partials in a fixed order and selects the heads); HISA
// reduces A over heads.  Both are O(H * M * d) per query, a few
// percent of the token scoring, and run here on the fp32 CUDA cores with the
// query heads and a chunk of block means staged in shared memory.
#include "launch.h"
#include "misa_device.cuh"

namespace misa {

namespace {

constexpr int kThreads = 256;
constexpr int kChunk = 32;        // blocks per CTA (8 warps x 4 blocks)
constexpr int kPad = kD + 4;      // fp32 row pitch in shared memory (keeps float4 alignment, spreads banks)

// Selection of routing decision g by one CTA (kThreads threads): importance =
// sum of the partials of its queries and chunks in a fixed order (thread
// (part, head) sums every P-th partial, then warp 0 adds the P parts in order),
// then h rounds of warp arg-max (value desc, id asc), then the chosen ids in
// ascending order.
__device__ void select_heads(const float* __restrict__ partial, float* sred, int T, int H, int n_chunks, int q_block,
                             int g, int h, int32_t* __restrict__ heads, float* __restrict__ importance) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int t0 = g * q_block;
  const int t1 = (t0 + q_block < T) ? t0 + q_block : T;
  const int n_pairs = (t1 - t0) * n_chunks;
  const int P = kThreads / H;  // >= 2 since H <= 128
  if (tid < P * H) {
    const int hh = tid % H, part = tid / H;
    float s = 0.f;
    for (int x = part; x < n_pairs; x += P) {
      const int t = t0 + x / n_chunks, c = x % n_chunks;
      s += __ldcg(&partial[(static_cast<int64_t>(t) * n_chunks + c) * H + hh]);
    }
    sred[part * H + hh] = s;
  }
  __syncthreads();
  if (warp != 0) return;
  constexpr int kMaxHB = MISA_MAX_HEADS / 32;
  float imp[kMaxHB];
  bool taken[kMaxHB];
#pragma unroll
  for (int a = 0; a < kMaxHB; ++a) {
    const int hh = lane + 32 * a;
    float s = 0.f;
    if (hh < H) {
      for (int part = 0; part < P; ++part) s += sred[part * H + hh];
      if (importance) importance[static_cast<int64_t>(g) * H + hh] = s;
    }
    imp[a] = s;
    taken[a] = false;
  }
  for (int r = 0; r < h; ++r) {
    float best = 0.f;
    int bid = 0x7fffffff;
#pragma unroll
    for (int a = 0; a < kMaxHB; ++a) {
      const int hh = lane + 32 * a;
      if (hh < H && !taken[a]) {
        if (bid == 0x7fffffff || imp[a] > best || (imp[a] == best && hh < bid)) {
          best = imp[a];
          bid = hh;
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ob = __shfl_xor_sync(0xffffffffu, best, o);
      const int oid = __shfl_xor_sync(0xffffffffu, bid, o);
      const bool better = (oid != 0x7fffffff) && (bid == 0x7fffffff || ob > best || (ob == best && oid < bid));
      if (better) {
        best = ob;
        bid = oid;
      }
    }
#pragma unroll
    for (int a = 0; a < kMaxHB; ++a)
      if (lane + 32 * a == bid) taken[a] = true;
  }
  // Ascending output: rank of a chosen head = chosen heads with a smaller id.
  int before = 0;
#pragma unroll
  for (int a = 0; a < kMaxHB; ++a) {
    const unsigned mask = __ballot_sync(0xffffffffu, taken[a]);
    if (taken[a]) {
      const int pos = before + __popc(mask & ((1u << lane) - 1u));
      heads[static_cast<int64_t>(g) * h + pos] = lane + 32 * a;
    }
    before += __popc(mask);
  }
}

// grid: (T, n_chunks).  Thread (warp jq, lane hp) owns heads hp + 32*a and
// blocks chunk*32 + 4*jq + u (u < 4).
template <bool kHisa>
__global__ void __launch_bounds__(kThreads)
affinity_kernel(const uint16_t* __restrict__ q, const float* __restrict__ w, const float* __restrict__ means,
                int64_t means_seq_stride, const int32_t* __restrict__ seq_of, const int32_t* __restrict__ prefix_len,
                int T, int H, int64_t L, int B, int M, int q_block, int nseq_means,
                float* __restrict__ partial,  // router: [T][n_chunks][H]
                unsigned* __restrict__ counters,  // router: [G] CTAs finished per decision (zero on entry)
                int h, int32_t* __restrict__ heads, float* __restrict__ importance,
                float* __restrict__ bscore,   // HISA:   [T][bs_stride]
                int64_t bs_stride,
                uint32_t* __restrict__ err) {
  extern __shared__ float4 smem_f4[];
  float* sq = reinterpret_cast<float*>(smem_f4);   // [H][kPad]
  float* sm = sq + H * kPad;                        // [kChunk][kPad]
  float* sred = sm + kChunk * kPad;                 // [8][H] (router) or unused
  __shared__ float sw[MISA_MAX_HEADS];

  const int t = blockIdx.x;
  const int chunk = blockIdx.y;
  const int n_chunks = gridDim.y;
  const int tid = threadIdx.x;
  const int lane = tid & 31;
  const int jq = tid >> 5;

  int seq = seq_of[t];
  if (seq < 0 || seq >= nseq_means) {
    if (tid == 0) record_error(err, MISA_DEVERR_BAD_SEQ);
    seq = 0;
  }
  // Visibility: a block is seen iff it lies wholly inside the prefix of the
  // query that owns the decision (the first query of its query block).
  const int t_dec = kHisa ? t : (t / q_block) * q_block;
  const int64_t plen = prefix_len[t_dec];

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

  if constexpr (!kHisa) {
    // Router: sum over this thread's 4 blocks, then over the 8 warps.
#pragma unroll
    for (int a = 0; a < kMaxHB; ++a) {
      const int h = lane + 32 * a;
      if (a < HB && h < H) sred[jq * H + h] = ((acc[a][0] + acc[a][1]) + acc[a][2]) + acc[a][3];
    }
    __syncthreads();
    for (int hh = tid; hh < H; hh += kThreads) {
      float s = 0.f;
#pragma unroll
      for (int k = 0; k < kThreads / 32; ++k) s += sred[k * H + hh];
      partial[(static_cast<int64_t>(t) * n_chunks + chunk) * H + hh] = s;
    }
    // The last CTA of this routing decision to finish selects its heads.
    __shared__ unsigned s_last;
    const int g = t / q_block;
    const int tq0 = g * q_block;
    const int tq1 = (tq0 + q_block < T) ? tq0 + q_block : T;
    __threadfence();
    __syncthreads();
    if (tid == 0) {
      const unsigned expected = static_cast<unsigned>((tq1 - tq0) * n_chunks);
      const unsigned old = atomicAdd(&counters[g], 1u);
      s_last = (old + 1u == expected) ? 1u : 0u;
    }
    __syncthreads();
    if (s_last) {
      __threadfence();
      select_heads(partial, sred, T, H, n_chunks, q_block, g, h, heads, importance);
      if (tid == 0) counters[g] = 0u;  // leave the counter ready for the next call
    }
  } else {
    // HISA: block score = sum over heads (this thread's heads, then the warp).
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      float s = 0.f;
#pragma unroll
      for (int a = 0; a < kMaxHB; ++a) s += acc[a][u];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      const int j = chunk * kChunk + jq * 4 + u;
      if (lane == 0 && j < M) bscore[static_cast<int64_t>(t) * bs_stride + j] = vis[u] ? s : -__int_as_float(0x7f800000);
    }
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

size_t affinity_smem_bytes(int H) {
  const int red = 8 * H > kThreads ? 8 * H : kThreads;  // per-warp sums, then the selection's partial sums
  return static_cast<size_t>(H * kPad + kChunk * kPad + red) * sizeof(float);
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

cudaError_t launch_route_heads(const uint16_t* q, const float* w, const float* means, int64_t means_seq_stride,
                               const int32_t* seq_of, const int32_t* prefix_len, int T, int H, int64_t L, int B,
                               int q_block, int h, int nseq_means, int32_t* heads, float* importance, float* partial,
                               unsigned* counters, uint32_t* err, cudaStream_t stream) {
  const int M = static_cast<int>((L + B - 1) / B);
  const int nch = router_chunks(M);
  const int G = (T + q_block - 1) / q_block;
  cudaError_t e = cudaMemsetAsync(counters, 0, static_cast<size_t>(G) * sizeof(unsigned), stream);
  if (e != cudaSuccess) return e;
  const size_t smem = affinity_smem_bytes(H);
  e = ensure_dynamic_smem(reinterpret_cast<const void*>(affinity_kernel<false>), static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  affinity_kernel<false><<<dim3(T, nch), kThreads, smem, stream>>>(q, w, means, means_seq_stride, seq_of, prefix_len,
                                                                   T, H, L, B, M, q_block, nseq_means, partial,
                                                                   counters, h, heads, importance, nullptr, 0, err);
  return cudaGetLastError();
}

cudaError_t launch_hisa_block_scores(const uint16_t* q, const float* w, const float* means, int64_t means_seq_stride,
                                     const int32_t* seq_of, const int32_t* prefix_len, int T, int H, int64_t L, int B,
                                     int nseq_means, float* bscore, int64_t bs_stride, uint32_t* err,
                                     cudaStream_t stream) {
  const int M = static_cast<int>((L + B - 1) / B);
  const int nch = router_chunks(M);
  const size_t smem = affinity_smem_bytes(H);
  cudaError_t e = ensure_dynamic_smem(reinterpret_cast<const void*>(affinity_kernel<true>), static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  affinity_kernel<true><<<dim3(T, nch), kThreads, smem, stream>>>(q, w, means, means_seq_stride, seq_of, prefix_len, T,
                                                                  H, L, B, M, 1, nseq_means, nullptr, nullptr, 0,
                                                                  nullptr, nullptr, bscore, bs_stride, err);
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
