// Head router on the 5th-generation tensor cores.
//
// "MISA: Mixture of Indexer Sparse Attention for Long-Context LLM Inference"
// (gist.science), Methodology: per-head affinities against block-aggregated
// keys are aggregated into an importance per head for the current query (block)
// and the top-h heads are kept.
//
//   importance[g][h] = sum over the queries t of decision g, and over the blocks
//                      j visible to g, of w[t][h] * ReLU(q[t][h] . mean_j)
//
// The contraction q . mean_j for all (query, head) rows and all blocks is an MMA:
// M = 128 (query, head) rows of one sequence (qpm queries x H heads, zero rows
// past them), N = 128 blocks per tile, K = 128.  The fp32 block means are split
// on the fly into bf16 hi = bf16(m) and lo = bf16(m - hi) (together about 16
// significant bits), and D = q . hi + q . lo accumulates in fp32 in TMEM.  The
// epilogue thread of row (t, h) sums ReLU(D) over the visible blocks of the tile
// in registers and over the tiles of its row group, then multiplies by w[t][h]:
// no cross-thread reduction.  A decision's rows are combined in shared memory;
// when a decision spans several row groups (prefill), the last CTA to finish
// one of them (atomic counter) sums the groups' partials in a fixed order.
// The top-h selection (ties to the lower head id, ids ascending) is one warp.
//
// Roles (288 threads): warps 0-3 epilogue (TMEM lane quarter = warp), warp 4
// TMEM allocation + MMA issue, warps 5-8 producers (query rows once per row
// group; block-mean tiles converted to hi/lo each tile).  Waits are bounded.
#include <algorithm>

#include "launch.h"
#include "misa_device.cuh"

namespace misa {

namespace {

constexpr int kRM = 128;                       // MMA M: (query, head) rows
constexpr int kRN = 128;                       // MMA N: blocks per tile
constexpr int kRStages = 2;
constexpr int kREpiThreads = 128;
constexpr int kRProdThreads = 128;
constexpr int kRMmaWarp = 4;
constexpr int kRProdWarp0 = 5;
constexpr int kRThreads = 288;
constexpr int kRATileBytes = kRM * kD * 2;     // 32 KB of query rows
constexpr int kRBTileBytes = kRN * kD * 2;     // 32 KB per hi or lo tile
constexpr int kRStageBytes = 2 * kRBTileBytes;
constexpr int kRTmemCols = 2 * kRN;            // two accumulators
constexpr uint32_t kRIdesc = idesc_bf16_f32(kRM, kRN);
constexpr int kROffA = 0;
constexpr int kROffB = kRATileBytes;
constexpr int kROffBar = kROffB + kRStages * kRStageBytes;
constexpr int kRNumBars = 2 * kRStages + 2 + 2 + 3;
constexpr int kROffTmem = kROffBar + kRNumBars * 8;
constexpr int kROffRed = (kROffTmem + 4 + 15) / 16 * 16;       // [128] row sums
constexpr int kROffImp = kROffRed + kRM * 4;                     // [MISA_MAX_HEADS] decision importances
constexpr int kROffFlag = kROffImp + MISA_MAX_HEADS * 4;
constexpr int kRSmemBytes = kROffFlag + 16 + 1024;

struct RouteParams {
  const uint16_t* q;
  const float* w;
  const float* means;
  int64_t means_seq_stride;
  int nseq;
  const int32_t* seq_of;
  const int32_t* prefix_len;
  int T, H;
  int64_t L;
  int B, M, q_block, h;
  int qpm;        // queries per row group (share one sequence and one decision)
  int n_pg;       // row groups
  int n_bt;       // block tiles
  float* partial;            // [n_pg][H] row-group importances (decisions spanning several groups)
  unsigned* counters;        // [G] groups finished per decision (zero on entry)
  int32_t* heads;            // [G][h]
  float* importance;         // [G][H] or NULL
  uint32_t* err;
};

__device__ __forceinline__ int group_seq(const RouteParams& p, int pg) {
  int seq = p.seq_of[pg * p.qpm];
  if (seq < 0 || seq >= p.nseq) {
    record_error(p.err, MISA_DEVERR_BAD_SEQ);
    seq = 0;
  }
  return seq;
}

// number of blocks visible to decision g (whole blocks inside the prefix of its first query)
__device__ __forceinline__ int visible_blocks(const RouteParams& p, int g) {
  const int64_t pl = p.prefix_len[static_cast<int64_t>(g) * p.q_block];
  if (pl >= p.L) return p.M;
  if (pl <= 0) return 0;
  return static_cast<int>(pl / p.B);
}

// Top-h of imp[0, H) (value desc, id asc), ids ascending into heads[g]; one warp.
__device__ void select_top_h(const float* imp, int H, int h, int g, int32_t* heads, float* importance) {
  const int lane = threadIdx.x & 31;
  constexpr int kMaxHB = MISA_MAX_HEADS / 32;
  float v[kMaxHB];
  bool taken[kMaxHB];
#pragma unroll
  for (int a = 0; a < kMaxHB; ++a) {
    const int hh = lane + 32 * a;
    v[a] = hh < H ? imp[hh] : 0.f;
    taken[a] = false;
    if (importance && hh < H) importance[static_cast<int64_t>(g) * H + hh] = v[a];
  }
  for (int r = 0; r < h; ++r) {
    float best = 0.f;
    int bid = 0x7fffffff;
#pragma unroll
    for (int a = 0; a < kMaxHB; ++a) {
      const int hh = lane + 32 * a;
      if (hh < H && !taken[a] && (bid == 0x7fffffff || v[a] > best || (v[a] == best && hh < bid))) {
        best = v[a];
        bid = hh;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ob = __shfl_xor_sync(0xffffffffu, best, o);
      const int oid = __shfl_xor_sync(0xffffffffu, bid, o);
      if (oid != 0x7fffffff && (bid == 0x7fffffff || ob > best || (ob == best && oid < bid))) {
        best = ob;
        bid = oid;
      }
    }
#pragma unroll
    for (int a = 0; a < kMaxHB; ++a)
      if (lane + 32 * a == bid) taken[a] = true;
  }
  int before = 0;
#pragma unroll
  for (int a = 0; a < kMaxHB; ++a) {
    const unsigned mask = __ballot_sync(0xffffffffu, taken[a]);
    if (taken[a]) heads[static_cast<int64_t>(g) * h + before + __popc(mask & ((1u << lane) - 1u))] = lane + 32 * a;
    before += __popc(mask);
  }
}

__global__ void __launch_bounds__(kRThreads, 1) route_tc_kernel(const RouteParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem + kROffA;
  uint8_t* sB = smem + kROffB;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kROffBar);
  uint64_t* full = bars;
  uint64_t* empty = bars + kRStages;
  uint64_t* tfull = bars + 2 * kRStages;
  uint64_t* tempty = bars + 2 * kRStages + 2;
  uint64_t* afull = bars + 2 * kRStages + 4;
  uint64_t* aempty = bars + 2 * kRStages + 5;
  uint64_t* done = bars + 2 * kRStages + 6;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kROffTmem);
  float* red = reinterpret_cast<float*>(smem + kROffRed);
  float* imp = reinterpret_cast<float*>(smem + kROffImp);
  unsigned* flag = reinterpret_cast<unsigned*>(smem + kROffFlag);
  volatile uint32_t* abort = reinterpret_cast<volatile uint32_t*>(smem + kROffFlag + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < kRStages; ++s) {
      mbar_init(&full[s], kRProdThreads);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], kREpiThreads);
    }
    mbar_init(afull, kRProdThreads);
    mbar_init(aempty, 1);
    mbar_init(done, 1);
    *abort = 0u;
    fence_mbar_init();
  }
  if (warp == kRMmaWarp) {
    tmem_alloc(tmem_slot, kRTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  // this CTA's row groups (whole groups, so the block sums stay in registers)
  const int pg0 = static_cast<int>(static_cast<int64_t>(p.n_pg) * blockIdx.x / gridDim.x);
  const int pg1 = static_cast<int>(static_cast<int64_t>(p.n_pg) * (blockIdx.x + 1) / gridDim.x);

  if (warp >= kRProdWarp0) {
    // ------------------------------------------------------------ producers
    const int pt = tid - kRProdWarp0 * 32;
    int64_t it = 0;
    bool ok = true;
    for (int pg = pg0, ng = 0; pg < pg1 && ok; ++pg, ++ng) {
      // query rows of the group: row r = ql * H + hh
      if (ng > 0 && !mbar_wait(aempty, (ng - 1) & 1, p.err, abort)) break;
      for (int x = pt; x < kRM * 16; x += kRProdThreads) {
        const int r = x >> 4, ch = x & 15;
        const int ql = r / p.H, hh = r - ql * p.H;
        const int t = pg * p.qpm + ql;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (ql < p.qpm && t < p.T)
          v = __ldg(reinterpret_cast<const uint4*>(p.q + (static_cast<int64_t>(t) * p.H + hh) * kD + ch * 8));
        *reinterpret_cast<uint4*>(sA + sw128_tile_offset(kRM, r, ch)) = v;
      }
      fence_proxy_async_smem();
      mbar_arrive(afull);
      const float* mb = p.means + static_cast<int64_t>(group_seq(p, pg)) * p.means_seq_stride;
      for (int bt = 0; bt < p.n_bt; ++bt, ++it) {
        const int s = static_cast<int>(it % kRStages);
        const uint32_t ph = static_cast<uint32_t>((it / kRStages) & 1);
        if (!mbar_wait(&empty[s], ph ^ 1u, p.err, abort)) { ok = false; break; }
        uint8_t* hi_t = sB + s * kRStageBytes;
        uint8_t* lo_t = hi_t + kRBTileBytes;
        // 128 blocks x 16 chunks of 8 means; 4 chunks in flight per thread
        for (int x0 = pt; x0 < kRN * 16; x0 += 4 * kRProdThreads) {
          float4 f[4][2];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int x = x0 + u * kRProdThreads;
            const int r = x >> 4, ch = x & 15;
            const int j = bt * kRN + r;
            if (x < kRN * 16 && j < p.M) {
              const float4* src = reinterpret_cast<const float4*>(mb + static_cast<int64_t>(j) * kD + ch * 8);
              f[u][0] = __ldg(src);
              f[u][1] = __ldg(src + 1);
            } else {
              f[u][0] = f[u][1] = make_float4(0.f, 0.f, 0.f, 0.f);
            }
          }
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int x = x0 + u * kRProdThreads;
            if (x >= kRN * 16) continue;
            const int r = x >> 4, ch = x & 15;
            const float e[8] = {f[u][0].x, f[u][0].y, f[u][0].z, f[u][0].w,
                                f[u][1].x, f[u][1].y, f[u][1].z, f[u][1].w};
            uint32_t hw[4], lw[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const __nv_bfloat16 h0 = __float2bfloat16_rn(e[2 * c]);
              const __nv_bfloat16 h1 = __float2bfloat16_rn(e[2 * c + 1]);
              const __nv_bfloat16 l0 = __float2bfloat16_rn(e[2 * c] - __bfloat162float(h0));
              const __nv_bfloat16 l1 = __float2bfloat16_rn(e[2 * c + 1] - __bfloat162float(h1));
              hw[c] = static_cast<uint32_t>(__bfloat16_as_ushort(h0)) |
                      (static_cast<uint32_t>(__bfloat16_as_ushort(h1)) << 16);
              lw[c] = static_cast<uint32_t>(__bfloat16_as_ushort(l0)) |
                      (static_cast<uint32_t>(__bfloat16_as_ushort(l1)) << 16);
            }
            const uint32_t off = sw128_tile_offset(kRN, r, ch);
            *reinterpret_cast<uint4*>(hi_t + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
            *reinterpret_cast<uint4*>(lo_t + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
          }
        }
        fence_proxy_async_smem();
        mbar_arrive(&full[s]);
      }
    }
  } else if (warp == kRMmaWarp) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      int64_t it = 0;
      const uint32_t a_addr = smem_u32(sA);
      bool ok = true;
      for (int pg = pg0, ng = 0; pg < pg1 && ok; ++pg, ++ng) {
        if (!mbar_wait(afull, ng & 1, p.err, abort)) break;
        for (int bt = 0; bt < p.n_bt; ++bt, ++it) {
          const int a = static_cast<int>(it & 1);
          const uint32_t aph = static_cast<uint32_t>((it >> 1) & 1);
          if (!mbar_wait(&tempty[a], aph ^ 1u, p.err, abort)) { ok = false; break; }
          const int s = static_cast<int>(it % kRStages);
          const uint32_t ph = static_cast<uint32_t>((it / kRStages) & 1);
          if (!mbar_wait(&full[s], ph, p.err, abort)) { ok = false; break; }
          tc_fence_after();
          const uint32_t hi_addr = smem_u32(sB + s * kRStageBytes);
          const uint32_t lo_addr = hi_addr + kRBTileBytes;
          const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(a * kRN);
#pragma unroll
          for (int kk = 0; kk < kD / 16; ++kk) {
            const uint32_t koff = (kk >> 2) * (kRM * 128) + (kk & 3) * 32;
            const uint32_t boff = (kk >> 2) * (kRN * 128) + (kk & 3) * 32;
            const uint64_t adesc = sw128_kmajor_desc(a_addr + koff);
            umma_bf16(d_tmem, adesc, sw128_kmajor_desc(hi_addr + boff), kRIdesc, kk > 0 ? 1u : 0u);
            umma_bf16(d_tmem, adesc, sw128_kmajor_desc(lo_addr + boff), kRIdesc, 1u);
          }
          umma_commit(&empty[s]);
          if (bt + 1 == p.n_bt) umma_commit(aempty);
          umma_commit(&tfull[a]);
        }
      }
      umma_commit(done);
      mbar_wait(done, 0, p.err);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int r = warp * 32 + lane;  // row (ql, hh) of the group
    const uint32_t t_lane = tmem_base + (static_cast<uint32_t>(warp * 32) << 16);
    // After a wait gives up the loops keep running without work ("skip"), so
    // every epilogue thread still reaches every named barrier.
    int64_t it = 0;
    bool skip = false;
    for (int pg = pg0; pg < pg1; ++pg) {
      const int g = (pg * p.qpm) / p.q_block;
      const int nvis = visible_blocks(p, g);
      float rowsum = 0.f;
      for (int bt = 0; bt < p.n_bt; ++bt, ++it) {
        const int a = static_cast<int>(it & 1);
        const uint32_t aph = static_cast<uint32_t>((it >> 1) & 1);
        if (skip || !mbar_wait(&tfull[a], aph, p.err, abort)) {
          skip = true;
          continue;
        }
        tc_fence_after();
        int nc = nvis - bt * kRN;  // visible columns of this tile
        nc = nc < 0 ? 0 : (nc > kRN ? kRN : nc);
        const uint32_t t_acc = t_lane + static_cast<uint32_t>(a * kRN);
        float s = 0.f;
#pragma unroll
        for (int c0 = 0; c0 < kRN; c0 += 64) {
          uint32_t v[64];
#pragma unroll
          for (int u = 0; u < 4; ++u) tmem_ld16(t_acc + static_cast<uint32_t>(c0 + 16 * u), v + 16 * u);
          tmem_wait_ld();
          if (c0 + 64 == kRN) {
            tc_fence_before();
            mbar_arrive(&tempty[a]);
          }
          if (c0 + 64 <= nc) {
#pragma unroll
            for (int jj = 0; jj < 64; ++jj) s += fmaxf(__uint_as_float(v[jj]), 0.f);
          } else {
#pragma unroll
            for (int jj = 0; jj < 64; ++jj) s += (c0 + jj < nc) ? fmaxf(__uint_as_float(v[jj]), 0.f) : 0.f;
          }
        }
        rowsum += s;
      }
      // row (t, hh) importance contribution, combined over the group's queries
      const int ql = r / p.H, hh = r - ql * p.H;
      const int t = pg * p.qpm + ql;
      float contrib = 0.f;
      if (ql < p.qpm && t < p.T) contrib = p.w[static_cast<int64_t>(t) * p.H + hh] * rowsum;
      red[r] = contrib;
      named_bar_sync(1, kREpiThreads);
      const int pgs_per_dec = p.q_block / p.qpm;  // row groups of a full decision
      const int first_pg = g * pgs_per_dec;
      const int last_pg = (first_pg + pgs_per_dec < p.n_pg ? first_pg + pgs_per_dec : p.n_pg) - 1;
      if (first_pg == last_pg) {
        // the whole decision is this group: select here
        if (tid < p.H) {
          float sum = 0.f;
          for (int k2 = 0; k2 < p.qpm; ++k2) sum += red[k2 * p.H + tid];
          imp[tid] = sum;
        }
        named_bar_sync(1, kREpiThreads);
        if (warp == 0 && !*abort) select_top_h(imp, p.H, p.h, g, p.heads, p.importance);
      } else {
        if (tid < p.H) {
          float sum = 0.f;
          for (int k2 = 0; k2 < p.qpm; ++k2) sum += red[k2 * p.H + tid];
          p.partial[static_cast<int64_t>(pg) * p.H + tid] = sum;
        }
        __threadfence();
        named_bar_sync(1, kREpiThreads);
        if (tid == 0) {
          const unsigned expected = static_cast<unsigned>(last_pg - first_pg + 1);
          flag[0] = (!*abort && atomicAdd(&p.counters[g], 1u) + 1u == expected) ? 1u : 0u;
        }
        named_bar_sync(1, kREpiThreads);
        if (flag[0]) {
          __threadfence();
          if (tid < p.H) {
            float sum = 0.f;
            for (int x = first_pg; x <= last_pg; ++x) sum += __ldcg(&p.partial[static_cast<int64_t>(x) * p.H + tid]);
            imp[tid] = sum;
          }
          named_bar_sync(1, kREpiThreads);
          if (warp == 0) select_top_h(imp, p.H, p.h, g, p.heads, p.importance);
          if (tid == 0) p.counters[g] = 0u;  // ready for the next call
        }
      }
      named_bar_sync(1, kREpiThreads);  // red / imp / flag are reused by the next group
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kRMmaWarp) tmem_dealloc(tmem_base, kRTmemCols);
}

}  // namespace

int route_tc_queries_per_group(int H, int q_block, bool shared_sequence) {
  if (!shared_sequence) return 1;
  int qpm = 1;
  while (qpm * 2 * H <= kRM && q_block % (qpm * 2) == 0) qpm *= 2;
  return qpm;
}

size_t route_tc_partial_floats(int T, int H, int qpm) {
  return static_cast<size_t>((T + qpm - 1) / qpm) * H;
}

cudaError_t launch_route_heads_tc(const uint16_t* q, const float* w, const float* means, int64_t means_seq_stride,
                                  int nseq, const int32_t* seq_of, const int32_t* prefix_len, int T, int H, int64_t L,
                                  int B, int q_block, int h, int qpm, int32_t* heads, float* importance,
                                  float* partial, unsigned* counters, uint32_t* err, cudaStream_t stream) {
  RouteParams p;
  p.q = q;
  p.w = w;
  p.means = means;
  p.means_seq_stride = means_seq_stride;
  p.nseq = nseq;
  p.seq_of = seq_of;
  p.prefix_len = prefix_len;
  p.T = T;
  p.H = H;
  p.L = L;
  p.B = B;
  p.M = static_cast<int>((L + B - 1) / B);
  p.q_block = q_block;
  p.h = h;
  p.qpm = qpm;
  p.n_pg = (T + qpm - 1) / qpm;
  p.n_bt = (p.M + kRN - 1) / kRN;
  p.partial = partial;
  p.counters = counters;
  p.heads = heads;
  p.importance = importance;
  p.err = err;
  const int G = (T + q_block - 1) / q_block;
  cudaError_t e = cudaMemsetAsync(counters, 0, static_cast<size_t>(G) * sizeof(unsigned), stream);
  if (e != cudaSuccess) return e;
  e = ensure_dynamic_smem(reinterpret_cast<const void*>(route_tc_kernel), kRSmemBytes);
  if (e != cudaSuccess) return e;
  const int sms = device_sm_count();
  if (sms <= 0) return cudaErrorInvalidDevice;
  const int grid = std::max(1, std::min(p.n_pg, sms));
  route_tc_kernel<<<grid, kRThreads, kRSmemBytes, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace misa
