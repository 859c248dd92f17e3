// Per-row top-k of fp32 scores by radix select.
//
// MISA forum thread (zingnex.cn), "DeepSeek稀疏注意力（DSA）的突破": the indexer
// keeps the most relevant token subset for the main attention.  HISA explainer
// (zhichai.net), section 二: the indexer picks the top-k tokens per query;
// section 四: its output is k token indices.
//
// Order: larger score first, ties to the lower position, -0.0 == +0.0, -inf
// (and NaN) never selected; the selected positions come out in ascending order,
// -1 padded when the row holds fewer than k selectable entries.
//
// One CTA (1024 threads) per row.  Scores are mapped to order-preserving
// uint32 keys and the k-th largest key tau is found digit by digit
// (12 + 10 + 10 bits):
//   pass 1  histogram of the top 12 bits over the row (shared-memory atomics);
//           the bin b1 holding the k-th largest key is found by a suffix scan;
//   pass 2  one ordered sweep of the row: keys above b1 (all selected, fewer
//           than k) go to list G, keys in b1 (the only undecided ones) go to
//           the candidate list C, both in position order;
//   refine  two 10-bit histogram rounds over C (in shared memory) give tau and
//           how many keys equal to tau are taken (the lowest positions);
//   merge   G and the chosen part of C are merged by position into the output.
// If b1 holds more candidates than shared memory takes (or k is large), the two
// refine rounds run over the row instead and a final ordered sweep writes the
// output.  The ordered sweeps are block-wide exclusive scans over chunks of
// 4096 consecutive entries, so selection order = position order.
#include "launch.h"
#include "misa_device.cuh"

namespace misa {

namespace {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;
constexpr int kChunkElems = 4 * kThreads;  // entries per ordered sweep step
constexpr int kBins1 = 4096;               // top 12 bits
constexpr int kBins2 = 1024;               // 10-bit digits
constexpr int kCap = 8192;                 // candidate list capacity (fast path)
constexpr int kFastMaxK = 8192;            // G + chosen C list capacity (fast path)

struct TopkSmem {
  uint32_t hist[kBins1];
  uint32_t warp_tot[kWarps];
  uint32_t bcast[8];
};
constexpr size_t kListsOff = (sizeof(TopkSmem) + 15) / 16 * 16;
constexpr size_t kSmemFast = kListsOff + kFastMaxK * 4 + kCap * 8;

__device__ __forceinline__ bool selectable(float v) { return v == v && v > -__int_as_float(0x7f800000); }

// Load the 4 entries [p, p+4) of the row (positions >= n give -inf).
__device__ __forceinline__ void load4(const float* row, int64_t p, int64_t n, float (&v)[4]) {
  if (p + 3 < n) {
    const float4 f = __ldg(reinterpret_cast<const float4*>(row + p));
    v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = (p + i < n) ? __ldg(row + p + i) : -__int_as_float(0x7f800000);
  }
}

// Block-wide exclusive scan of a packed counter (two 16-bit fields); returns
// this thread's exclusive prefix, and the block total in *total.
__device__ __forceinline__ uint32_t block_exclusive_scan(TopkSmem& sm, uint32_t x, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t inc = x;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += y;
  }
  if (lane == 31) sm.warp_tot[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    uint32_t t = sm.warp_tot[lane];
    uint32_t ti = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, ti, o);
      if (lane >= o) ti += y;
    }
    sm.warp_tot[lane] = ti - t;  // exclusive warp offsets
    if (lane == 31) sm.bcast[7] = ti;
  }
  __syncthreads();
  const uint32_t res = sm.warp_tot[warp] + inc - x;
  *total = sm.bcast[7];
  __syncthreads();  // warp_tot / bcast reused by the next scan
  return res;
}

// Find the bin holding the need-th largest key: bins [0, nbins) with counts
// in hist; returns bin b with sum(hist[b+1..]) < need <= sum(hist[b..]) and the
// count strictly above it in *above.  Requires 1 <= need <= total.
__device__ __forceinline__ int find_bin(TopkSmem& sm, int nbins, uint32_t need, uint32_t* above) {
  const int per = nbins / kThreads;  // 4 or 1
  const int b0 = threadIdx.x * per;
  uint32_t local = 0;
  for (int i = 0; i < per; ++i) local += sm.hist[b0 + i];
  // suffix sums over threads: scan in reversed thread order
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t inc = local;  // inclusive suffix within warp (lanes >= me)
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_down_sync(0xffffffffu, inc, o);
    if (lane + o < 32) inc += y;
  }
  if (lane == 0) sm.warp_tot[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    uint32_t t = sm.warp_tot[lane];
    uint32_t ti = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_down_sync(0xffffffffu, ti, o);
      if (lane + o < 32) ti += y;
    }
    sm.warp_tot[lane] = ti - t;  // suffix of the warps after this one
  }
  __syncthreads();
  // suffix strictly after this thread's bins
  uint32_t after = sm.warp_tot[warp] + inc - local;
  if (after < need && after + local >= need) {
    uint32_t acc = after;
    for (int i = per - 1; i >= 0; --i) {
      const uint32_t c = sm.hist[b0 + i];
      if (acc + c >= need) {
        sm.bcast[0] = static_cast<uint32_t>(b0 + i);
        sm.bcast[1] = acc;
        break;
      }
      acc += c;
    }
  }
  __syncthreads();
  const int bin = static_cast<int>(sm.bcast[0]);
  *above = sm.bcast[1];
  __syncthreads();
  return bin;
}

__device__ __forceinline__ void clear_hist(TopkSmem& sm, int nbins) {
  for (int i = threadIdx.x; i < nbins; i += kThreads) sm.hist[i] = 0;
  __syncthreads();
}

__device__ __forceinline__ int32_t out_id(const int32_t* idrow, int64_t pos) {
  return idrow ? idrow[pos] : static_cast<int32_t>(pos);
}

__global__ void __launch_bounds__(kThreads, 1)
topk_kernel(const float* __restrict__ scores, int64_t n, int64_t row_stride, const int32_t* __restrict__ row_valid,
            const int32_t* __restrict__ id_map, int64_t id_map_stride, int k, int32_t* __restrict__ idx) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  TopkSmem& sm = *reinterpret_cast<TopkSmem*>(smem_raw);
  int32_t* lists = reinterpret_cast<int32_t*>(smem_raw + kListsOff);   // G at [0, gt), chosen C at [gt, k)
  uint32_t* ckey = reinterpret_cast<uint32_t*>(lists + kFastMaxK);     // C keys
  int32_t* cpos = reinterpret_cast<int32_t*>(ckey + kCap);             // C positions

  const int t = blockIdx.x;
  const int tid = threadIdx.x;
  const float* row = scores + static_cast<int64_t>(t) * row_stride;
  const int32_t* idrow = id_map ? id_map + static_cast<int64_t>(t) * id_map_stride : nullptr;
  int32_t* out = idx + static_cast<int64_t>(t) * k;
  int64_t nt = n;
  if (row_valid) {
    const int64_t rv = row_valid[t];
    nt = rv < 0 ? 0 : (rv < n ? rv : n);
  }

  // ---------------- pass 1: top-12-bit histogram
  clear_hist(sm, kBins1);
  for (int64_t p = static_cast<int64_t>(tid) * 4; p < nt; p += kChunkElems) {
    float v[4];
    load4(row, p, nt, v);
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if (selectable(v[i])) atomicAdd(&sm.hist[float_key(v[i]) >> 20], 1u);
  }
  __syncthreads();
  uint32_t total = 0;
  {
    uint32_t local = 0;
    for (int i = tid * 4; i < tid * 4 + 4; ++i) local += sm.hist[i];
    block_exclusive_scan(sm, local, &total);
  }

  if (total <= static_cast<uint32_t>(k)) {
    // every selectable entry is chosen: one ordered sweep, then -1 padding
    uint32_t base = 0;
    for (int64_t c0 = 0; c0 < nt; c0 += kChunkElems) {
      const int64_t p = c0 + static_cast<int64_t>(tid) * 4;
      float v[4];
      load4(row, p, nt, v);
      uint32_t cnt = 0;
#pragma unroll
      for (int i = 0; i < 4; ++i) cnt += selectable(v[i]) ? 1u : 0u;
      uint32_t tot;
      uint32_t off = base + block_exclusive_scan(sm, cnt, &tot);
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (selectable(v[i])) out[off++] = out_id(idrow, p + i);
      base += tot;
    }
    for (int i = static_cast<int>(total) + tid; i < k; i += kThreads) out[i] = -1;
    return;
  }

  uint32_t gt1;
  const int b1 = find_bin(sm, kBins1, static_cast<uint32_t>(k), &gt1);
  const uint32_t cnt1 = sm.hist[b1];
  __syncthreads();

  if (k <= kFastMaxK && cnt1 <= static_cast<uint32_t>(kCap)) {
    // ---------------- pass 2: ordered split into G (bin > b1) and C (bin == b1)
    uint32_t gbase = 0, cbase = 0;
    for (int64_t c0 = 0; c0 < nt; c0 += kChunkElems) {
      const int64_t p = c0 + static_cast<int64_t>(tid) * 4;
      float v[4];
      load4(row, p, nt, v);
      uint32_t key[4];
      uint32_t packed = 0;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        key[i] = selectable(v[i]) ? float_key(v[i]) : 0u;
        const uint32_t bin = key[i] >> 20;
        if (key[i] && static_cast<int>(bin) > b1) packed += 1u;
        else if (key[i] && static_cast<int>(bin) == b1) packed += 1u << 16;
      }
      uint32_t tot;
      const uint32_t pre = block_exclusive_scan(sm, packed, &tot);
      uint32_t go = gbase + (pre & 0xffffu), co = cbase + (pre >> 16);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        if (!key[i]) continue;
        const int bin = static_cast<int>(key[i] >> 20);
        if (bin > b1) {
          lists[go++] = static_cast<int32_t>(p + i);
        } else if (bin == b1) {
          ckey[co] = key[i];
          cpos[co] = static_cast<int32_t>(p + i);
          ++co;
        }
      }
      gbase += tot & 0xffffu;
      cbase += tot >> 16;
    }
    __syncthreads();
    // ---------------- refine inside C
    const uint32_t need = static_cast<uint32_t>(k) - gt1;  // 1 <= need <= cnt1
    clear_hist(sm, kBins2);
    for (uint32_t i = tid; i < cnt1; i += kThreads) atomicAdd(&sm.hist[(ckey[i] >> 10) & 0x3ffu], 1u);
    __syncthreads();
    uint32_t gt2;
    const int b2 = find_bin(sm, kBins2, need, &gt2);
    const uint32_t need2 = need - gt2;
    clear_hist(sm, kBins2);
    for (uint32_t i = tid; i < cnt1; i += kThreads)
      if (static_cast<int>((ckey[i] >> 10) & 0x3ffu) == b2) atomicAdd(&sm.hist[ckey[i] & 0x3ffu], 1u);
    __syncthreads();
    uint32_t gt3;
    const int b3 = find_bin(sm, kBins2, need2, &gt3);
    const uint32_t need_eq = need2 - gt3;  // keys equal to tau to take, lowest positions first
    const uint32_t tau = (static_cast<uint32_t>(b1) << 20) | (static_cast<uint32_t>(b2) << 10) |
                         static_cast<uint32_t>(b3);
    // ordered compaction of the chosen candidates into lists[gt1 ..)
    {
      uint32_t sbase = 0, ebase = 0;
      for (uint32_t c0 = 0; c0 < cnt1; c0 += kChunkElems) {
        uint32_t packed = 0;
        uint32_t kk[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint32_t ci = c0 + tid * 4 + i;
          kk[i] = ci < cnt1 ? ckey[ci] : 0u;
          if (ci < cnt1) packed += (kk[i] > tau) ? 1u : ((kk[i] == tau) ? (1u << 16) : 0u);
        }
        uint32_t tot;
        const uint32_t pre = block_exclusive_scan(sm, packed, &tot);
        uint32_t so = sbase + (pre & 0xffffu), eo = ebase + (pre >> 16);
        // a key equal to tau is taken iff its rank among equal keys is < need_eq;
        // chosen entries keep position order: rank among chosen = (#above before) + min(#equal before, need_eq)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint32_t ci = c0 + tid * 4 + i;
          if (ci >= cnt1) continue;
          if (kk[i] > tau) {
            const uint32_t eq_before = eo < need_eq ? eo : need_eq;
            lists[gt1 + so + eq_before] = cpos[ci];
            ++so;
          } else if (kk[i] == tau) {
            if (eo < need_eq) lists[gt1 + so + eo] = cpos[ci];
            ++eo;
          }
        }
        sbase += tot & 0xffffu;
        ebase += tot >> 16;
      }
    }
    __syncthreads();
    // ---------------- merge G = lists[0, gt1) and chosen C = lists[gt1, k) by position
    const int32_t* G = lists;
    const int32_t* Cs = lists + gt1;
    const int nG = static_cast<int>(gt1), nC = k - static_cast<int>(gt1);
    for (int i = tid; i < nG; i += kThreads) {
      const int32_t pos = G[i];
      int lo = 0, hi = nC;  // count of Cs < pos
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (Cs[mid] < pos) lo = mid + 1; else hi = mid;
      }
      out[i + lo] = out_id(idrow, pos);
    }
    for (int i = tid; i < nC; i += kThreads) {
      const int32_t pos = Cs[i];
      int lo = 0, hi = nG;
      while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (G[mid] < pos) lo = mid + 1; else hi = mid;
      }
      out[i + lo] = out_id(idrow, pos);
    }
    return;
  }

  // ---------------- general path: refine over the row, then one ordered sweep
  const uint32_t need = static_cast<uint32_t>(k) - gt1;
  clear_hist(sm, kBins2);
  for (int64_t p = static_cast<int64_t>(tid) * 4; p < nt; p += kChunkElems) {
    float v[4];
    load4(row, p, nt, v);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      if (!selectable(v[i])) continue;
      const uint32_t key = float_key(v[i]);
      if (static_cast<int>(key >> 20) == b1) atomicAdd(&sm.hist[(key >> 10) & 0x3ffu], 1u);
    }
  }
  __syncthreads();
  uint32_t gt2;
  const int b2 = find_bin(sm, kBins2, need, &gt2);
  const uint32_t need2 = need - gt2;
  const uint32_t pre22 = (static_cast<uint32_t>(b1) << 10) | static_cast<uint32_t>(b2);
  clear_hist(sm, kBins2);
  for (int64_t p = static_cast<int64_t>(tid) * 4; p < nt; p += kChunkElems) {
    float v[4];
    load4(row, p, nt, v);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      if (!selectable(v[i])) continue;
      const uint32_t key = float_key(v[i]);
      if ((key >> 10) == pre22) atomicAdd(&sm.hist[key & 0x3ffu], 1u);
    }
  }
  __syncthreads();
  uint32_t gt3;
  const int b3 = find_bin(sm, kBins2, need2, &gt3);
  const uint32_t need_eq = need2 - gt3;
  const uint32_t tau = (pre22 << 10) | static_cast<uint32_t>(b3);
  uint32_t sbase = 0, ebase = 0;
  for (int64_t c0 = 0; c0 < nt; c0 += kChunkElems) {
    const int64_t p = c0 + static_cast<int64_t>(tid) * 4;
    float v[4];
    load4(row, p, nt, v);
    uint32_t key[4];
    uint32_t packed = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      key[i] = selectable(v[i]) ? float_key(v[i]) : 0u;
      packed += (key[i] > tau) ? 1u : ((key[i] && key[i] == tau) ? (1u << 16) : 0u);
    }
    uint32_t tot;
    const uint32_t pre = block_exclusive_scan(sm, packed, &tot);
    uint32_t so = sbase + (pre & 0xffffu), eo = ebase + (pre >> 16);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      if (key[i] > tau) {
        const uint32_t eq_before = eo < need_eq ? eo : need_eq;
        out[so + eq_before] = out_id(idrow, p + i);
        ++so;
      } else if (key[i] && key[i] == tau) {
        if (eo < need_eq) out[so + eo] = out_id(idrow, p + i);
        ++eo;
      }
    }
    sbase += tot & 0xffffu;
    ebase += tot >> 16;
  }
}

}  // namespace

size_t topk_smem_bytes() { return kSmemFast; }

cudaError_t launch_topk(const float* scores, int T, int64_t n, int64_t row_stride, const int32_t* row_valid,
                        const int32_t* id_map, int64_t id_map_stride, int k, int32_t* idx, cudaStream_t stream) {
  cudaError_t e = ensure_dynamic_smem(reinterpret_cast<const void*>(topk_kernel), static_cast<int>(kSmemFast));
  if (e != cudaSuccess) return e;
  topk_kernel<<<T, kThreads, kSmemFast, stream>>>(scores, n, row_stride, row_valid, id_map, id_map_stride, k, idx);
  return cudaGetLastError();
}

}  // namespace misa
