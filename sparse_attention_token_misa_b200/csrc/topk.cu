// Per-row top-k of fp32 scores.
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
// Four kernels, by row count and length (launch_topk):
//  * many rows (at least two per SM), up to 131072 entries: topk_band_kernel,
//    one CTA per row, a sampled band around the k-th entry;
//  * few rows of up to 8192 entries: topk_row_kernel, one CTA per row, the
//    row in registers, a value-range histogram;
//  * few rows of 8193 .. 131072 entries: topk_rowc_kernel, the same over a
//    cluster of up to 8 CTAs per row;
//  * few longer rows: topk_cluster_kernel, a cluster of 8 CTAs per row, the
//    k-th largest key digit by digit (12 + 10 + 10 bits): every CTA
//    histograms the digit over its slice, the histograms are summed through
//    distributed shared memory (each CTA owns 1/8 of the bins), every CTA
//    finds the bin holding the k-th key; ballots, a scan over the warps and
//    the per-CTA counts give every selected entry its slot.
// Each kernel's comment describes it.  In every kernel keys equal to the k-th
// largest are taken lowest position first, exactly as many as needed.
#include <cooperative_groups.h>

#include "launch.h"
#include "misa_device.cuh"

namespace cg = cooperative_groups;

namespace misa {

namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kBins1 = 4096;  // first digit: top 12 bits
constexpr int kBins2 = 1024;  // second and third digits: 10 bits each
constexpr int kMaxCluster = 8;

struct Smem {
  uint32_t hist[kBins1];   // local histogram, then the pulled cluster histogram
  uint32_t own[kBins1];    // this CTA's share of the summed histogram
  uint32_t warp_tot[kWarps];
  uint32_t bcast[4];
  alignas(8) uint32_t counts[2];  // (above tau, equal to tau) in this CTA's slice
  uint64_t warp_tot64[kWarps];
  uint64_t block_tot64;
};
constexpr size_t kClusterSmemBytes = (sizeof(Smem) + 15) / 16 * 16;   // topk_cluster_kernel's shared memory

__device__ __forceinline__ bool selectable(float v) { return v == v && v > -__int_as_float(0x7f800000); }

// key of a score, 0 for entries that can never be selected
__device__ __forceinline__ uint32_t sel_key(float v) { return selectable(v) ? float_key(v) : 0u; }

__device__ __forceinline__ float valid_or_neg_inf(float v) { return selectable(v) ? v : -__int_as_float(0x7f800000); }

__device__ __forceinline__ uint32_t block_sum(Smem& sm, uint32_t x) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  if (lane == 0) sm.warp_tot[warp] = x;
  __syncthreads();
  uint32_t s = 0;
  for (int i = 0; i < kWarps; ++i) s += sm.warp_tot[i];
  __syncthreads();
  return s;
}

// Exclusive scan over the block's warps of a pair of counts packed as
// (lo | hi << 32); every thread passes its warp's total (lane-uniform).
__device__ __forceinline__ uint64_t warp_exclusive_scan(Smem& sm, uint64_t warp_total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (lane == 0) sm.warp_tot64[warp] = warp_total;
  __syncthreads();
  if (warp == 0) {
    const uint64_t tw = lane < kWarps ? sm.warp_tot64[lane] : 0ull;
    uint64_t ti = tw;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint64_t y = __shfl_up_sync(0xffffffffu, ti, o);
      if (lane >= o) ti += y;
    }
    if (lane < kWarps) sm.warp_tot64[lane] = ti - tw;
    if (lane == kWarps - 1) sm.block_tot64 = ti;
  }
  __syncthreads();
  const uint64_t res = sm.warp_tot64[warp];
  return res;
}

// In the (already summed) histogram hist[0, nbins): the bin b with
// sum(hist[b+1..]) < need <= sum(hist[b..]); *above = sum(hist[b+1..]).
__device__ __forceinline__ int find_bin(Smem& sm, int nbins, uint32_t need, uint32_t* above) {
  const int per = nbins / kThreads;  // 8 or 2
  const int b0 = threadIdx.x * per;
  uint32_t local = 0;
  for (int i = 0; i < per; ++i) local += sm.hist[b0 + i];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t inc = local;  // suffix over lanes >= me
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_down_sync(0xffffffffu, inc, o);
    if (lane + o < 32) inc += y;
  }
  if (lane == 0) sm.warp_tot[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    const uint32_t tw = lane < kWarps ? sm.warp_tot[lane] : 0u;
    uint32_t ti = tw;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_down_sync(0xffffffffu, ti, o);
      if (lane + o < 32) ti += y;
    }
    if (lane < kWarps) sm.warp_tot[lane] = ti - tw;  // suffix of later warps
  }
  __syncthreads();
  const uint32_t after = sm.warp_tot[warp] + inc - local;
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

// Sum the CL local histograms (hist, nbins) across the cluster and leave the
// summed histogram in every CTA's hist.  Two cluster barriers.
__device__ __forceinline__ void cluster_hist_sum(cg::cluster_group& cl, Smem& sm, int nbins, int CL, int rank) {
  cl.sync();  // every local histogram is complete
  const int share = nbins / CL;
  const int base = rank * share;
  for (int i = threadIdx.x; i < share; i += kThreads) {
    uint32_t x[kMaxCluster];  // all reads issued before the first is used
#pragma unroll
    for (int c = 0; c < kMaxCluster; ++c) x[c] = c < CL ? cl.map_shared_rank(&sm.hist[0], c)[base + i] : 0u;
    uint32_t s = 0;
#pragma unroll
    for (int c = 0; c < kMaxCluster; ++c) s += x[c];
    sm.own[i] = s;
  }
  cl.sync();  // every share is summed; local histograms are no longer read remotely
  for (int i = threadIdx.x; i < nbins; i += kThreads) {
    const int owner = i / share;
    sm.hist[i] = cl.map_shared_rank(&sm.own[0], owner)[i - owner * share];
  }
  __syncthreads();
}

__global__ void __launch_bounds__(kThreads, 2)
topk_cluster_kernel(const float* __restrict__ scores, int64_t n, int64_t row_stride, const int32_t* __restrict__ row_valid,
                    const int32_t* __restrict__ id_map, int64_t id_map_stride, int k, int32_t* __restrict__ idx,
                    int64_t slice_len) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>(smem_raw);

  pdl_wait_inputs();
  pdl_allow_next();
  cg::cluster_group cl = cg::this_cluster();
  const int CL = static_cast<int>(cl.num_blocks());
  const int rank = static_cast<int>(cl.block_rank());
  const int tid = threadIdx.x;
  const int64_t t = blockIdx.y;

  const float* row = scores + t * row_stride;
  const int32_t* idrow = id_map ? id_map + t * id_map_stride : nullptr;
  int32_t* out = idx + t * k;
  int64_t nt = n;
  if (row_valid) {
    const int64_t rv = row_valid[t];
    nt = rv < 0 ? 0 : (rv < n ? rv : n);
  }
  const int64_t s0 = rank * slice_len < nt ? rank * slice_len : nt;
  const int64_t s1 = s0 + slice_len < nt ? s0 + slice_len : nt;
  const int len = static_cast<int>(s1 - s0);

  // (the slices of rows this long do not fit in shared memory: every pass
  // reads its keys from global memory, where L2 keeps them)
  auto key_at = [&](int i) -> uint32_t { return sel_key(__ldg(row + s0 + i)); };

  // ---------------- digit 1 (top 12 bits) while loading the slice
  for (int i = tid; i < kBins1; i += kThreads) sm.hist[i] = 0;
  __syncthreads();
  {
    // 16-byte loads where the slice start is aligned (row_stride % 4 == 0 and
    // slices are multiples of 4 long), a scalar tail otherwise
    const int nv = len / 4;
    const float4* r4 = reinterpret_cast<const float4*>(row + s0);
    for (int i0 = tid; i0 < nv; i0 += 4 * kThreads) {
      float4 f[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = i0 + u * kThreads;
        f[u] = i < nv ? __ldg(r4 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = i0 + u * kThreads;
        if (i < nv) {
          const uint32_t kk[4] = {sel_key(f[u].x), sel_key(f[u].y), sel_key(f[u].z), sel_key(f[u].w)};
#pragma unroll
          for (int e = 0; e < 4; ++e)
            if (kk[e]) atomicAdd(&sm.hist[kk[e] >> 20], 1u);
        }
      }
    }
    for (int i = 4 * nv + tid; i < len; i += kThreads) {
      const uint32_t kk = sel_key(__ldg(row + s0 + i));
      if (kk) atomicAdd(&sm.hist[kk >> 20], 1u);
    }
  }
  __syncthreads();
  cluster_hist_sum(cl, sm, kBins1, CL, rank);
  uint32_t total = 0;
  {
    uint32_t local = 0;
    for (int i = tid; i < kBins1; i += kThreads) local += sm.hist[i];
    total = block_sum(sm, local);
  }

  uint32_t tau;       // selected: key > tau, or key == tau among the first need_eq
  uint32_t need_eq;
  if (total <= static_cast<uint32_t>(k)) {
    tau = kNegInfKey;  // every selectable key is above it
    need_eq = 0;
  } else {
    uint32_t gt1, gt2, gt3;
    const int b1 = find_bin(sm, kBins1, static_cast<uint32_t>(k), &gt1);
    const uint32_t need1 = static_cast<uint32_t>(k) - gt1;
    // ---------------- digit 2 (bits 19..10) among keys in bin b1
    for (int i = tid; i < kBins2; i += kThreads) sm.hist[i] = 0;
    __syncthreads();
    for (int i = tid; i < len; i += kThreads) {
      const uint32_t kk = key_at(i);
      if (kk && static_cast<int>(kk >> 20) == b1) atomicAdd(&sm.hist[(kk >> 10) & 0x3ffu], 1u);
    }
    __syncthreads();
    cluster_hist_sum(cl, sm, kBins2, CL, rank);
    const int b2 = find_bin(sm, kBins2, need1, &gt2);
    const uint32_t need2 = need1 - gt2;
    const uint32_t pre22 = (static_cast<uint32_t>(b1) << 10) | static_cast<uint32_t>(b2);
    // ---------------- digit 3 (bits 9..0) among keys with the 22-bit prefix
    for (int i = tid; i < kBins2; i += kThreads) sm.hist[i] = 0;
    __syncthreads();
    for (int i = tid; i < len; i += kThreads) {
      const uint32_t kk = key_at(i);
      if (kk && (kk >> 10) == pre22) atomicAdd(&sm.hist[kk & 0x3ffu], 1u);
    }
    __syncthreads();
    cluster_hist_sum(cl, sm, kBins2, CL, rank);
    const int b3 = find_bin(sm, kBins2, need2, &gt3);
    tau = (pre22 << 10) | static_cast<uint32_t>(b3);
    need_eq = need2 - gt3;
  }

  // ---------------- emission: warp w owns the contiguous chunk
  // [w * chunk, (w + 1) * chunk) of the slice and walks it 32 keys at a time
  // (lanes on consecutive keys, ballots give the in-warp order)
  const int lane = tid & 31, warp = tid >> 5;
  const int chunk = ((len + kWarps - 1) / kWarps + 31) / 32 * 32;
  const int c0 = warp * chunk < len ? warp * chunk : len;
  const int c1 = c0 + chunk < len ? c0 + chunk : len;
  uint32_t a_cnt = 0, e_cnt = 0;
  for (int i = c0 + lane; i < c1; i += 32) {
    const uint32_t kk = key_at(i);
    a_cnt += kk > tau ? 1u : 0u;
    e_cnt += (kk && kk == tau) ? 1u : 0u;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    a_cnt += __shfl_xor_sync(0xffffffffu, a_cnt, o);
    e_cnt += __shfl_xor_sync(0xffffffffu, e_cnt, o);
  }
  const uint64_t wpre = warp_exclusive_scan(sm, static_cast<uint64_t>(a_cnt) | (static_cast<uint64_t>(e_cnt) << 32));
  if (tid == 0) {
    sm.counts[0] = static_cast<uint32_t>(sm.block_tot64 & 0xffffffffull);
    sm.counts[1] = static_cast<uint32_t>(sm.block_tot64 >> 32);
  }
  cl.sync();  // per-CTA counts visible cluster-wide
  uint32_t a_before = 0, e_before = 0, a_all = 0, e_all = 0;
  uint2 cc[kMaxCluster];  // all reads issued before the first is used
#pragma unroll
  for (int c = 0; c < kMaxCluster; ++c)
    cc[c] = c < CL ? *reinterpret_cast<const uint2*>(cl.map_shared_rank(&sm.counts[0], c)) : make_uint2(0u, 0u);
#pragma unroll
  for (int c = 0; c < kMaxCluster; ++c) {
    if (c < rank) {
      a_before += cc[c].x;
      e_before += cc[c].y;
    }
    a_all += cc[c].x;
    e_all += cc[c].y;
  }
  cl.sync();  // no CTA reads another's shared memory after this point
  uint32_t a_pos = a_before + static_cast<uint32_t>(wpre & 0xffffffffull);
  uint32_t e_pos = e_before + static_cast<uint32_t>(wpre >> 32);
  const uint32_t lt = (1u << lane) - 1u;
  for (int i0 = c0; i0 < c1; i0 += 32) {
    const int i = i0 + lane;
    const uint32_t kk = i < c1 ? key_at(i) : 0u;
    const bool is_a = kk > tau;
    const bool is_e = kk && kk == tau;
    const uint32_t ba = __ballot_sync(0xffffffffu, is_a);
    const uint32_t be = __ballot_sync(0xffffffffu, is_e);
    const uint32_t my_a = a_pos + __popc(ba & lt);
    const uint32_t my_e = e_pos + __popc(be & lt);
    // slots are < k by construction; the bound check only guards the output
    if (is_a) {
      const uint32_t slot = my_a + (my_e < need_eq ? my_e : need_eq);
      if (slot < static_cast<uint32_t>(k)) out[slot] = idrow ? idrow[s0 + i] : static_cast<int32_t>(s0 + i);
    } else if (is_e && my_e < need_eq && my_a + my_e < static_cast<uint32_t>(k)) {
      out[my_a + my_e] = idrow ? idrow[s0 + i] : static_cast<int32_t>(s0 + i);
    }
    a_pos += __popc(ba);
    e_pos += __popc(be);
  }
  // -1 padding after the selected entries (only when fewer than k are selectable)
  if (rank == CL - 1) {
    const uint32_t chosen = a_all + (e_all < need_eq ? e_all : need_eq);
    for (uint32_t i = chosen + tid; i < static_cast<uint32_t>(k); i += kThreads) out[i] = -1;
  }
}

__device__ __forceinline__ float key_to_float(uint32_t kk) {
  const uint32_t u = (kk & 0x80000000u) ? (kk ^ 0x80000000u) : ~kk;
  return __uint_as_float(u);
}

// ---------------------------------------------------------------------------
// One CTA of 512 threads per row, no cluster (topk_band_kernel), rows of up
// to 131072 entries.  A sample of the row (4096 entries: 1024 evenly spaced
// groups of 4 adjacent ones) gives two thresholds lo <= hi that bracket the k-th largest entry with a
// wide margin: the sample is binned over its value range (4096 equal ranges,
// a monotone map); the bins holding sample ranks r - d and r + d (r the rank
// the k-th entry has in the sample on average, d = 3 sqrt(r) + 8) give hi (the
// largest sample value not above the upper bin) and lo (the smallest sample
// value not below the lower bin).  One pass over the row (128-entry steps
// dealt round-robin to the warps, lane l reading entries 32 c + l so that one
// ballot is one bitmap word) writes a bitmap of the entries above hi, counts
// them, and gathers the band [lo, hi] with positions into per-warp buffers.
// When the band holds the k-th entry, a radix select over the gathered
// entries gives the exact threshold tau and the band entries above / equal to
// it join the bitmaps; otherwise (the sample misled, too many ties to gather,
// or fewer valid entries than k) a radix select over the whole row gives tau
// and one more pass rebuilds the bitmaps.  The output comes from the bitmaps:
// per-warp counts, a scan over the warps and over each warp's words give every
// selected position its slot, so the row is read once on the common path.
constexpr int kBThreads = 512;
constexpr int kBWarps = kBThreads / 32;
constexpr int kBSample = 4096;
constexpr int kBBins = 4096;
constexpr int kBWarpCap = 384;                  // band entries kept per warp
constexpr int kBCandCap = kBWarpCap * kBWarps;  // 6144
constexpr int kBMaxN = 131072;                  // longest row (bitmaps in shared memory)
constexpr int kBWords = kBMaxN / 32 + kBWarps * 4;  // + segment rounding
#ifndef MISA_BAND_UNROLL
#define MISA_BAND_UNROLL 4
#endif
constexpr int kBUnroll = MISA_BAND_UNROLL;  // steps whose loads are in flight together per warp

constexpr int kBListCap = 256;  // band entries in one value-range bin ranked by counting

struct BSmem {
  uint32_t hist[kBBins];
  union {
    float sval[kBSample];     // the sample (until the thresholds are known)
    float cval[kBCandCap];    // then the band entries, kBWarpCap per warp,
  };
  int32_t cpos[kBCandCap];    // and their positions
  uint32_t gt[kBWords];     // bitmap: selected, above tau
  uint32_t eq[kBWords];     // bitmap: equal to tau
  uint32_t wa[kBWarps], wc[kBWarps];  // per warp: entries above hi, entries gathered
  uint32_t at[kBWarps], et[kBWarps];  // per warp: bits set in gt / eq
  uint32_t wtmp[kBWarps];
  uint32_t wend[kBWarps];             // per warp: end of its candidates in the flat order
  float wmin[kBWarps], wmax[kBWarps];
  uint32_t bc[8];
  float fbc[2];
  float lval[kBListCap];      // band entries in the bin of the k-th entry (range path)
  uint32_t lcnt;
};

// Over hist[0, nbins) (nbins a multiple of 512, <= 4096): for each of the two
// targets the bin b with above(b) < need <= above(b) + hist[b], above(b) = sum
// of the higher bins: out[0] = b, out[1] = above(b) for need1, out[2], out[3]
// for need2 (left unchanged when a target exceeds the total).  All threads.
__device__ __forceinline__ void band_find(BSmem& sm, const uint32_t* hist, int nbins, uint32_t need1,
                                          uint32_t need2, uint32_t* out) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int per = nbins / kBThreads;
  const int b0 = tid * per;
  uint32_t local = 0;
  for (int i = 0; i < per; ++i) local += hist[b0 + i];
  uint32_t inc = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_down_sync(0xffffffffu, inc, o);
    if (lane + o < 32) inc += y;
  }
  if (lane == 0) sm.wtmp[warp] = inc;
  __syncthreads();
  uint32_t higher = 0;
#pragma unroll
  for (int w2 = 0; w2 < kBWarps; ++w2) higher += w2 > warp ? sm.wtmp[w2] : 0u;
  const uint32_t after = higher + inc - local;
  const uint32_t needs[2] = {need1, need2};
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    const uint32_t need = needs[q];
    if (after < need && need <= after + local) {
      uint32_t acc = after;
      for (int i = per - 1; i >= 0; --i) {
        const uint32_t c = hist[b0 + i];
        if (acc + c >= need) {
          out[2 * q] = static_cast<uint32_t>(b0 + i);
          out[2 * q + 1] = acc;
          break;
        }
        acc += c;
      }
    }
  }
  __syncthreads();
}

// Exact radix select (12 + 10 + 10 key bits) of the need-th largest key among
// the keys visit(fn) hands to fn (0 = not a candidate); returns its key and
// sets *gt to the number of larger keys.  All threads.
template <class Visit>
__device__ uint32_t band_radix_visit(BSmem& sm, Visit visit, uint32_t need, uint32_t* gt) {
  const int tid = threadIdx.x;
  uint32_t prefix = 0, above = 0;
  for (int round = 0; round < 3; ++round) {
    const int sh = round == 0 ? 20 : (round == 1 ? 10 : 0);
    const int nb = round == 0 ? 4096 : 1024;
    for (int i = tid; i < nb; i += kBThreads) sm.hist[i] = 0;
    __syncthreads();
    visit([&](uint32_t kk) {
      if (kk == 0u) return;
      const bool match = round == 0 || (kk >> (round == 1 ? 20 : 10)) == prefix;
      if (match) atomicAdd(&sm.hist[(kk >> sh) & static_cast<uint32_t>(nb - 1)], 1u);
    });
    __syncthreads();
    band_find(sm, sm.hist, nb, need, 0xffffffffu, sm.bc);
    const uint32_t b = sm.bc[0] & static_cast<uint32_t>(nb - 1);
    const uint32_t ab = sm.bc[1];
    __syncthreads();
    above += ab;
    need -= ab;
    prefix = round == 0 ? b : ((prefix << 10) | b);
  }
  *gt = above;
  return prefix;
}

// The same over key_at(i), 0 <= i < n_keys.
template <class KeyAt>
__device__ uint32_t band_radix(BSmem& sm, int n_keys, KeyAt key_at, uint32_t need, uint32_t* gt) {
  return band_radix_visit(
      sm,
      [&](auto fn) {
        for (int i = threadIdx.x; i < n_keys; i += kBThreads) fn(key_at(i));
      },
      need, gt);
}

__global__ void __launch_bounds__(kBThreads, 2)
topk_band_kernel(const float* __restrict__ scores, int64_t n, int64_t row_stride, const int32_t* __restrict__ row_valid,
                 const int32_t* __restrict__ id_map, int64_t id_map_stride, int k, int32_t* __restrict__ idx) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  BSmem& sm = *reinterpret_cast<BSmem*>(smem_raw);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t t = blockIdx.x;
  const float kNegInf = -__int_as_float(0x7f800000);
  const float kPosInf = __int_as_float(0x7f800000);
  const float kLowest = -__int_as_float(0x7f7fffff);  // -FLT_MAX: v >= it iff v is selectable
  const uint32_t ku = static_cast<uint32_t>(k);

  pdl_wait_inputs();
  pdl_allow_next();
  const float* row = scores + t * row_stride;
  const int32_t* idrow = id_map ? id_map + t * id_map_stride : nullptr;
  int32_t* out = idx + t * k;
  int64_t nt64 = n;
  if (row_valid) {
    const int64_t rv = row_valid[t];
    nt64 = rv < 0 ? 0 : (rv < n ? rv : n);
  }
  const int nt = static_cast<int>(nt64);
  const int nsteps = (nt + 127) / 128;  // 128-entry steps; warp w takes steps w, w + 16, ...
  auto load_step = [&](int base, float x[4]) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int p = base + 32 * c + lane;
      x[c] = p < nt ? __ldg(row + p) : kNegInf;
    }
  };

  // ---------------- sample: value range, then its histogram.  Rows longer
  // than the sample give 1024 evenly spaced groups of 4 adjacent entries (one
  // 16-byte load each: a quarter of the DRAM bursts of 4096 scattered
  // entries); shorter rows are sampled whole.
  const int ns = nt < kBSample ? nt : kBSample;
  float mx = kNegInf, mn = kPosInf;
  {
    constexpr int kG = kBSample / 4 / kBThreads;  // groups per thread (2)
    float4 sv[kG];
#pragma unroll
    for (int u = 0; u < kG; ++u) {
      const int g = tid + u * kBThreads;  // group: sample entries 4 g .. 4 g + 3
      if (nt <= kBSample) {
        float e[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) e[j] = 4 * g + j < nt ? __ldg(row + 4 * g + j) : kNegInf;
        sv[u] = make_float4(e[0], e[1], e[2], e[3]);
      } else {
        const int p = static_cast<int>(static_cast<int64_t>(g) * nt / (kBSample / 4)) & ~3;
        sv[u] = p + 3 < nt ? __ldg(reinterpret_cast<const float4*>(row + p))
                           : make_float4(__ldg(row + p), p + 1 < nt ? __ldg(row + p + 1) : kNegInf,
                                         p + 2 < nt ? __ldg(row + p + 2) : kNegInf, kNegInf);
      }
    }
#pragma unroll
    for (int u = 0; u < kG; ++u) {
      const int g = tid + u * kBThreads;
      const float e[4] = {sv[u].x, sv[u].y, sv[u].z, sv[u].w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float v = valid_or_neg_inf(e[j]);
        if (4 * g + j < ns) sm.sval[4 * g + j] = v;
        if (v > kNegInf) {
          mx = fmaxf(mx, v);
          mn = fminf(mn, v);
        }
      }
    }
  }
  for (int i = tid; i < kBBins; i += kBThreads) sm.hist[i] = 0;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
  }
  if (lane == 0) {
    sm.wmax[warp] = mx;
    sm.wmin[warp] = mn;
  }
  __syncthreads();
  mx = sm.wmax[0];
  mn = sm.wmin[0];
#pragma unroll
  for (int i = 1; i < kBWarps; ++i) {
    mx = fmaxf(mx, sm.wmax[i]);
    mn = fminf(mn, sm.wmin[i]);
  }
  const float range = mx - mn;
  const float scale = (range > 0.f && range < kPosInf) ? static_cast<float>(kBBins) / range : 0.f;
  // monotone in x; a NaN intermediate (no valid sample, infinite entries) maps to bin 0
  auto bin_of = [&](float x) -> int {
    const float y = __fmul_rn(__fsub_rn(x, mn), scale);
    return y > 0.f ? (y >= static_cast<float>(kBBins - 1) ? kBBins - 1 : static_cast<int>(y)) : 0;
  };
  uint32_t nsv = 0;
  for (int i = tid; i < ns; i += kBThreads) {
    const float v = sm.sval[i];
    if (v > kNegInf) {
      atomicAdd(&sm.hist[bin_of(v)], 1u);
      ++nsv;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) nsv += __shfl_xor_sync(0xffffffffu, nsv, o);
  if (lane == 0) sm.wtmp[warp] = nsv;
  __syncthreads();
  nsv = 0;
#pragma unroll
  for (int i = 0; i < kBWarps; ++i) nsv += sm.wtmp[i];
  __syncthreads();
  // bins holding sample ranks r -/+ d (0-based, from the top)
  const int64_t r = static_cast<int64_t>(k) * ns / (nt > 0 ? nt : 1);
  const int64_t d = static_cast<int64_t>(3.f * sqrtf(static_cast<float>(r))) + 8;
  const int64_t r_hi = r - d, r_lo = r + d;
  if (tid == 0) {
    sm.bc[0] = kBBins;  // r_hi < 0: nothing lies above the band
    sm.bc[2] = 0;
  }
  __syncthreads();
  band_find(sm, sm.hist, kBBins, r_hi >= 0 ? static_cast<uint32_t>(r_hi + 1) : 0xffffffffu,
            r_lo < static_cast<int64_t>(nsv) ? static_cast<uint32_t>(r_lo + 1) : 0xffffffffu, sm.bc);
  const int b_hi = static_cast<int>(sm.bc[0]);
  const int b_lo = static_cast<int>(sm.bc[2]);
  // thresholds in value space: hi = the largest sample not above bin b_hi
  // (+inf when nothing lies above), lo = the smallest sample not below bin b_lo
  // (-FLT_MAX, every selectable entry, when r + d is past the valid sample)
  float hv = kNegInf, lv = kPosInf;
  for (int i = tid; i < ns; i += kBThreads) {
    const float v = sm.sval[i];
    if (v > kNegInf) {
      const int b = bin_of(v);
      if (b <= b_hi) hv = fmaxf(hv, v);
      if (b >= b_lo) lv = fminf(lv, v);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    hv = fmaxf(hv, __shfl_xor_sync(0xffffffffu, hv, o));
    lv = fminf(lv, __shfl_xor_sync(0xffffffffu, lv, o));
  }
  if (lane == 0) {
    sm.wmax[warp] = hv;
    sm.wmin[warp] = lv;
  }
  __syncthreads();
  hv = sm.wmax[0];
  lv = sm.wmin[0];
#pragma unroll
  for (int i = 1; i < kBWarps; ++i) {
    hv = fmaxf(hv, sm.wmax[i]);
    lv = fminf(lv, sm.wmin[i]);
  }
  const float hi_v = b_hi >= kBBins ? kPosInf : hv;
  const float lo_v = (r_lo >= static_cast<int64_t>(nsv) || !(lv <= hi_v)) ? kLowest : lv;

  // ---------------- pass 1 (the only read of the row on the common path):
  // lane l of a warp holds positions 128 st + 4 l .. 4 l + 3 of step st (one
  // 16-byte load); the 32 positions of bitmap word q of the step are held by
  // lanes 8 q .. 8 q + 7, four bits each, OR-ed together over those lanes
  if (lane == 0) sm.wc[warp] = 0u;
  __syncwarp();
  uint32_t a_l = 0;  // entries above hi seen by this lane
  float* wcval = sm.cval + warp * kBWarpCap;
  int32_t* wcpos = sm.cpos + warp * kBWarpCap;
  for (int s0 = warp; s0 < nsteps; s0 += kBWarps * kBUnroll) {
    float4 xs[kBUnroll];
#pragma unroll
    for (int u = 0; u < kBUnroll; ++u) {
      const int p = 128 * (s0 + kBWarps * u) + 4 * lane;
      if (p + 3 < nt) {
        xs[u] = __ldg(reinterpret_cast<const float4*>(row + p));
      } else {
        xs[u].x = p < nt ? __ldg(row + p) : kNegInf;
        xs[u].y = p + 1 < nt ? __ldg(row + p + 1) : kNegInf;
        xs[u].z = p + 2 < nt ? __ldg(row + p + 2) : kNegInf;
        xs[u].w = kNegInf;
      }
    }
#pragma unroll
    for (int u = 0; u < kBUnroll; ++u) {
      const int st = s0 + kBWarps * u;
      if (st >= nsteps) break;
      const float e[4] = {xs[u].x, xs[u].y, xs[u].z, xs[u].w};
      uint32_t anib = 0u, bnib = 0u;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const bool above = e[c] > hi_v;            // false for NaN
        const bool band = !above && e[c] >= lo_v;  // false for NaN and -inf
        anib |= above ? 1u << c : 0u;
        bnib |= band ? 1u << c : 0u;
      }
      uint32_t aw = anib << (4 * (lane & 7));
      aw |= __shfl_xor_sync(0xffffffffu, aw, 1);
      aw |= __shfl_xor_sync(0xffffffffu, aw, 2);
      aw |= __shfl_xor_sync(0xffffffffu, aw, 4);
      if ((lane & 7) == 0) sm.gt[4 * st + (lane >> 3)] = aw;
      a_l += static_cast<uint32_t>(__popc(anib));
      if (bnib) {
        uint32_t sl = atomicAdd(&sm.wc[warp], static_cast<uint32_t>(__popc(bnib)));
#pragma unroll
        for (int c = 0; c < 4; ++c)
          if ((bnib >> c) & 1u) {
            if (sl < static_cast<uint32_t>(kBWarpCap)) {
              wcval[sl] = e[c];
              wcpos[sl] = 128 * st + 4 * lane + c;
            }
            ++sl;
          }
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) a_l += __shfl_xor_sync(0xffffffffu, a_l, o);
  if (lane == 0) sm.wa[warp] = a_l;
  // the equal-to-tau bitmap starts empty
  const int nwords = nsteps * 4;
  for (int i = tid; i < nwords; i += kBThreads) sm.eq[i] = 0u;
  __syncthreads();
  uint32_t A = 0, C = 0;
  bool full = false;
#pragma unroll
  for (int i = 0; i < kBWarps; ++i) {
    A += sm.wa[i];
    C += sm.wc[i];
    full |= sm.wc[i] > static_cast<uint32_t>(kBWarpCap);
  }

  float tau;
  uint32_t need_eq;
  if (A < ku && ku <= A + C && !full) {
    // the k-th entry is in the band (so at least k entries are selectable):
    // exact tau among the gathered entries, which then join the bitmaps
    // the warps' filled candidate slots as one flat range: region ends in
    // registers, a flat index mapped to (region, slot) by compares
    if (tid < kBWarps) {
      uint32_t e = 0;
      for (int w2 = 0; w2 <= tid; ++w2) e += sm.wc[w2];
      sm.wend[tid] = e;
    }
    __syncthreads();
    auto each_cand = [&](auto fn) {
      for (uint32_t f = tid; f < C; f += kBThreads) {
        int slot = static_cast<int>(f);
#pragma unroll
        for (int w2 = 0; w2 < kBWarps - 1; ++w2) {
          const uint32_t e = sm.wend[w2];
          if (f >= e) slot = (w2 + 1) * kBWarpCap + static_cast<int>(f - e);
        }
        fn(slot);
      }
    };
    // tau: a histogram of the band entries over their own value range (2048
    // equal-width bins, monotone in the value), then the entries of the bin
    // holding the k-th one ranked by counting; radix rounds over the band
    // entries when the range is degenerate or that bin is crowded (ties)
    uint32_t gt = 0;
    bool resolved = false;
    {
      float cmn = kPosInf, cmx = kNegInf;
      each_cand([&](int i) {
        cmn = fminf(cmn, sm.cval[i]);
        cmx = fmaxf(cmx, sm.cval[i]);
      });
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        cmn = fminf(cmn, __shfl_xor_sync(0xffffffffu, cmn, o));
        cmx = fmaxf(cmx, __shfl_xor_sync(0xffffffffu, cmx, o));
      }
      __syncthreads();   // wmin / wmax were read by every thread before
      if (lane == 0) {
        sm.wmin[warp] = cmn;
        sm.wmax[warp] = cmx;
      }
      for (int i = tid; i < 2048; i += kBThreads) sm.hist[i] = 0u;
      if (tid == 0) sm.lcnt = 0u;
      __syncthreads();
      cmn = sm.wmin[0];
      cmx = sm.wmax[0];
#pragma unroll
      for (int i = 1; i < kBWarps; ++i) {
        cmn = fminf(cmn, sm.wmin[i]);
        cmx = fmaxf(cmx, sm.wmax[i]);
      }
      const float span = cmx - cmn;
      const float cscale = 2048.f / span;
      const float coff = -cmn * cscale;
      if (cmx > cmn && span > 0.f && isfinite(span) && isfinite(cscale) && isfinite(coff)) {   // (CTA-uniform)
        auto cbin = [&](float x) {
          const float y = fminf(fmaxf(fmaf(x, cscale, coff), 0.f), 2047.f) + 8388608.f;
          return __float_as_uint(y) & 2047u;
        };
        each_cand([&](int i) { atomicAdd(&sm.hist[cbin(sm.cval[i])], 1u); });
        __syncthreads();
        band_find(sm, sm.hist, 2048, ku - A, 0xffffffffu, sm.bc);
        const uint32_t bstar = sm.bc[0] & 2047u;
        const uint32_t above_b = sm.bc[1];
        const uint32_t c = sm.hist[bstar];
        if (c <= static_cast<uint32_t>(kBListCap)) {   // (CTA-uniform)
          each_cand([&](int i) {
            const float x = sm.cval[i];
            if (cbin(x) == bstar) {
              const uint32_t s2 = atomicAdd(&sm.lcnt, 1u);
              if (s2 < static_cast<uint32_t>(kBListCap)) sm.lval[s2] = x;
            }
          });
          __syncthreads();
          const uint32_t need2 = ku - A - above_b;   // 1 <= need2 <= c
          if (static_cast<uint32_t>(tid) < c) {
            const float x = sm.lval[tid];
            uint32_t g2 = 0, eb = 0;
            for (uint32_t j = 0; j < c; ++j) {
              const float y = sm.lval[j];
              g2 += y > x ? 1u : 0u;
              eb += (y == x && j < static_cast<uint32_t>(tid)) ? 1u : 0u;
            }
            if (g2 + eb == need2 - 1u) {
              sm.fbc[0] = x;
              sm.bc[4] = g2;
            }
          }
          __syncthreads();
          tau = sm.fbc[0];
          gt = above_b + sm.bc[4];
          resolved = true;
        }
      }
    }
    if (!resolved) {
      const uint32_t kk = band_radix_visit(
          sm, [&](auto fn) { each_cand([&](int i) { fn(float_key(sm.cval[i])); }); }, ku - A, &gt);
      tau = key_to_float(kk);
    }
    need_eq = ku - A - gt;
    each_cand([&](int i) {
      const float x = sm.cval[i];
      const int p = sm.cpos[i];
      if (x > tau) atomicOr(&sm.gt[p >> 5], 1u << (p & 31));
      else if (x == tau) atomicOr(&sm.eq[p >> 5], 1u << (p & 31));
    });
  } else {
    // the sample misled, too many ties to gather, or fewer selectable entries
    // than k: count the selectable entries; exact tau by a radix select over
    // the row when there are more than k; one more pass rebuilds the bitmaps
    uint32_t nv = 0;
    for (int st = warp; st < nsteps; st += kBWarps) {
      float x[4];
      load_step(128 * st, x);
#pragma unroll
      for (int c = 0; c < 4; ++c) nv += __popc(__ballot_sync(0xffffffffu, x[c] >= kLowest));
    }
    if (lane == 0) sm.wtmp[warp] = nv;
    __syncthreads();
    nv = 0;
#pragma unroll
    for (int i = 0; i < kBWarps; ++i) nv += sm.wtmp[i];
    __syncthreads();
    if (nv <= ku) {
      tau = kNegInf;  // every selectable entry
      need_eq = 0;
    } else {
      uint32_t gt;
      const uint32_t kk = band_radix(sm, nt, [&](int i) { return sel_key(__ldg(row + i)); }, ku, &gt);
      tau = key_to_float(kk);
      need_eq = ku - gt;
    }
    for (int st = warp; st < nsteps; st += kBWarps) {
      float x[4];
      load_step(128 * st, x);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const float v = valid_or_neg_inf(x[c]);
        const uint32_t gm = __ballot_sync(0xffffffffu, v > tau);
        const uint32_t em = __ballot_sync(0xffffffffu, v > kNegInf && v == tau);
        if (lane == 0) {
          sm.gt[4 * st + c] = gm;
          sm.eq[4 * st + c] = em;
        }
      }
    }
  }
  __syncthreads();

  // ---------------- per-warp counts from the bitmaps, then the output: warp w
  // owns a contiguous range of bitmap words and walks it 32 words at a time
  // (one per lane); a scan over the lanes gives each word's first slot
  const int wpw = (nsteps * 4 + kBWarps - 1) / kBWarps;
  const int wd0 = warp * wpw < nsteps * 4 ? warp * wpw : nsteps * 4;
  const int wd1 = wd0 + wpw < nsteps * 4 ? wd0 + wpw : nsteps * 4;
  {
    uint32_t g = 0, e = 0;
    for (int i = wd0 + lane; i < wd1; i += 32) {
      g += __popc(sm.gt[i]);
      e += __popc(sm.eq[i]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      g += __shfl_xor_sync(0xffffffffu, g, o);
      e += __shfl_xor_sync(0xffffffffu, e, o);
    }
    if (lane == 0) {
      sm.at[warp] = g;
      sm.et[warp] = e;
    }
  }
  __syncthreads();
  uint32_t Aw = 0, Ew = 0, a_all = 0, e_all = 0;
#pragma unroll
  for (int i = 0; i < kBWarps; ++i) {
    const uint32_t ai = sm.at[i], ei = sm.et[i];
    Aw += i < warp ? ai : 0u;
    Ew += i < warp ? ei : 0u;
    a_all += ai;
    e_all += ei;
  }
  const uint32_t chosen = a_all + (e_all < need_eq ? e_all : need_eq);
  for (int i0 = wd0; i0 < wd1 && Aw < ku; i0 += 32) {
    const int i = i0 + lane;
    const uint32_t gw = i < wd1 ? sm.gt[i] : 0u;
    const uint32_t ew = i < wd1 ? sm.eq[i] : 0u;
    const uint32_t packed = static_cast<uint32_t>(__popc(gw)) | (static_cast<uint32_t>(__popc(ew)) << 16);
    uint32_t incl = packed;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const uint32_t tot = __shfl_sync(0xffffffffu, incl, 31);
    uint32_t a_pos = Aw + ((incl - packed) & 0xffffu);
    uint32_t e_pos = Ew + ((incl - packed) >> 16);
    uint32_t bits = gw | ew;
    while (bits) {
      const int bit = __ffs(bits) - 1;
      bits &= bits - 1;
      const int p = i * 32 + bit;
      if ((gw >> bit) & 1u) {
        const uint32_t slot = a_pos + (e_pos < need_eq ? e_pos : need_eq);
        if (slot < ku) out[slot] = idrow ? idrow[p] : p;
        ++a_pos;
      } else {
        if (e_pos < need_eq && a_pos + e_pos < ku) out[a_pos + e_pos] = idrow ? idrow[p] : p;
        ++e_pos;
      }
    }
    Aw += tot & 0xffffu;
    Ew += tot >> 16;
  }
  for (uint32_t i = chosen + tid; i < ku; i += kBThreads) out[i] = -1;
}

// ---------------------------------------------------------------------------
// Rows of up to 8192 entries, few rows (topk_row_kernel): one CTA of 1024
// threads per row, no cluster.  Warp w holds positions [w 32V, (w+1) 32V) of
// the row in registers (V = 4 or 8 per thread, loaded as coalesced float4:
// in step i lane l holds positions w 32V + 128 i + 4 l + (0..3)), so the row
// is read once and every later step is a pass over registers:
//   (1) a value range from a sample (each thread's first entry: 1024 evenly
//       spaced positions);
//   (2) a histogram over 2048 equal-width bins of that range (entries outside
//       it go to the end bins; the bin of a value is monotone in the value)
//       gives the selectable count, the bin b* holding the k-th largest entry
//       and the count above b*;
//   (3) one pass marks the entries above b* and lists those in b* (few, as a
//       rule) in shared memory; each listed entry's rank (value descending,
//       position ascending) is counted against the others, and the need
//       best-ranked ones are marked in their owner thread's mask;
//   (4) every thread writes its marked positions into slots from a scan over
//       the warp (per step) and over the warps, in position order.
// Values are compared as floats: NaN fails every test (never selected), -0.0
// equals +0.0.  General path, for a degenerate range or a long list: the
// exact k-th largest key tau by three radix rounds (11, 11, 10 key bits) over
// the list or over the registers, then the entries above tau and the lowest-
// position entries equal to it.
constexpr int kRThreads = 1024;
constexpr int kRWarps = kRThreads / 32;
constexpr int kRBins = 2048;
constexpr int kRCandCap = 4096;   // entries of b* listed in shared memory
constexpr int kRRankMax = 128;    // lists this short are ranked by counting

struct alignas(16) RSmem {
  uint32_t hist[kRBins];
  float cv[kRCandCap];        // the listed entries of b* and their positions
  int32_t cp[kRCandCap];
  uint32_t extra[kRThreads];  // per thread: listed entries that are selected (bit j)
  uint32_t red[3][kRWarps];   // scan scratch (halves 0 and 1 alternate), reductions
  uint32_t bc[2];
  uint32_t ccount;
  float tau;
  uint32_t take, eqtot;
};

// Exclusive scan of x over the CTA's 1024 threads, with red (32 words) as
// scratch; *total = the sum.  Alternating two scratch arrays, two scans in a
// row need no barrier between them.
__device__ __forceinline__ uint32_t cta_excl_scan(uint32_t x, uint32_t* red, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t inc = x;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += y;
  }
  if (lane == 31) red[warp] = inc;
  __syncthreads();
  const uint32_t wv = red[lane];
  uint32_t winc = wv;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, winc, o);
    if (lane >= o) winc += y;
  }
  const uint32_t before = __shfl_sync(0xffffffffu, winc - wv, warp);
  *total = __shfl_sync(0xffffffffu, winc, 31);
  return before + inc - x;
}

// The bin of h[0, nb) (nb = 1024 or 2048) holding the need-th largest entry:
// bc[0] = bin, bc[1] = entries in higher bins (set only when need <= the
// total).  Returns the histogram's total.  All 1024 threads; ends with a
// barrier.
__device__ __forceinline__ uint32_t cta_find_bin(const uint32_t* h, int nb, uint32_t need, uint32_t* red,
                                                 uint32_t* bc) {
  const int per = nb / kRThreads;
  const int b0 = threadIdx.x * per;
  uint32_t local = 0;
  for (int i = 0; i < per; ++i) local += h[b0 + i];
  uint32_t total;
  const uint32_t excl = cta_excl_scan(local, red, &total);
  const uint32_t after = total - excl - local;   // entries in the bins of higher threads
  if (after < need && need <= after + local) {
    uint32_t acc = after;
    for (int i = per - 1; i >= 0; --i) {
      const uint32_t c = h[b0 + i];
      if (acc + c >= need) {
        bc[0] = static_cast<uint32_t>(b0 + i);
        bc[1] = acc;
        break;
      }
      acc += c;
    }
  }
  __syncthreads();
  return total;
}

__device__ __forceinline__ uint32_t row_find_bin(RSmem& sm, int nb, uint32_t need, int buf) {
  return cta_find_bin(sm.hist, nb, need, sm.red[buf], sm.bc);
}

// Three radix rounds (11, 11, 10 key bits): the need-th largest key among the
// keys add_round(prefix, pmask, shift, nbins) counts into hist.  Leaves tau,
// take (entries equal to tau taken) and eqtot (entries equal to tau) in sm.
template <class AddRound>
__device__ __forceinline__ void row_radix(RSmem& sm, uint32_t need, AddRound add_round) {
  const int tid = threadIdx.x;
  uint32_t prefix = 0u, pmask = 0u, eqtot = 0u;
#pragma unroll 1
  for (int round = 0; round < 3; ++round) {
    const int sh = round == 0 ? 21 : (round == 1 ? 10 : 0);
    const int nb = round == 2 ? 1024 : 2048;
    __syncthreads();   // the previous readers of hist / bc are done
    for (int i = tid; i < nb; i += kRThreads) sm.hist[i] = 0u;
    __syncthreads();
    add_round(prefix, pmask, sh, nb);
    __syncthreads();
    row_find_bin(sm, nb, need, round & 1);
    const uint32_t d = sm.bc[0];
    need -= sm.bc[1];
    prefix |= d << sh;
    pmask |= static_cast<uint32_t>(nb - 1) << sh;
    if (round == 2) eqtot = sm.hist[d];
  }
  __syncthreads();
  if (tid == 0) {
    sm.tau = key_to_float(prefix);
    sm.take = need;
    sm.eqtot = eqtot;
  }
  __syncthreads();
}

// For each warp: the exclusive prefix of its total over the lower warps, and
// *all = the sum over the CTA.  x: this warp's total (same in every lane);
// red: 32 words of scratch.
__device__ __forceinline__ uint32_t cta_warp_base(uint32_t x, uint32_t* red, uint32_t* all) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (lane == 0) red[warp] = x;
  __syncthreads();
  const uint32_t wv = red[lane];
  uint32_t winc = wv;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, winc, o);
    if (lane >= o) winc += y;
  }
  *all = __shfl_sync(0xffffffffu, winc, 31);
  return __shfl_sync(0xffffffffu, winc - wv, warp);
}

__device__ __forceinline__ uint32_t row_warp_base(RSmem& sm, uint32_t x, int buf, uint32_t* all) {
  return cta_warp_base(x, sm.red[buf], all);
}

__device__ __forceinline__ uint32_t warp_sum(uint32_t x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// Entries are held as in topk_row_kernel: bit j of a thread's mask is its
// entry j, at position base + 128 (j / 4) + 4 lane + j % 4 of its warp's chunk.
//
// Of the entries marked in tk, the first `take` in position order over the
// CTA (warps in order, then steps, lanes, entries).  All threads.
template <int V>
__device__ __forceinline__ uint32_t cta_keep_first(uint32_t tk, uint32_t take, uint32_t* red) {
  const int lane = threadIdx.x & 31;
  const uint32_t lt = (1u << lane) - 1u;
  uint32_t all;
  uint32_t run = cta_warp_base(warp_sum(__popc(tk)), red, &all);
  uint32_t keep = 0u;
#pragma unroll
  for (int i = 0; i < V / 4; ++i) {
    uint32_t before = 0u, tot = 0u;
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {
      const uint32_t b = __ballot_sync(0xffffffffu, (tk >> (4 * i + cc)) & 1u);
      before += __popc(b & lt);
      tot += __popc(b);
    }
    uint32_t r = run + before;
#pragma unroll
    for (int cc = 0; cc < 4; ++cc)
      if ((tk >> (4 * i + cc)) & 1u) {
        if (r < take) keep |= 1u << (4 * i + cc);
        ++r;
      }
    run += tot;
  }
  return keep;
}

// Writes the entries marked in selm to out[base + slot] (through idrow when
// given), slots in position order over the CTA; per step i (4 entries per
// lane) the lane counts are packed in 8-bit fields (a warp's step total is
// <= 128).  Slots at or past ku are not written.  Returns the CTA's count.
// All threads.
template <int V, class PosOf>
__device__ __forceinline__ uint32_t cta_write_selected(uint32_t selm, uint32_t base, PosOf pos_of,
                                                       const int32_t* __restrict__ idrow, int32_t* __restrict__ out,
                                                       uint32_t ku, uint32_t* red) {
  static_assert(V <= 32, "eight steps at most");
  const int lane = threadIdx.x & 31;
  uint32_t plo = 0u, phi = 0u;
#pragma unroll
  for (int i = 0; i < V / 4; ++i) {
    const uint32_t cnt = static_cast<uint32_t>(__popc((selm >> (4 * i)) & 0xFu));
    if (i < 4) plo |= cnt << (8 * i);
    else phi |= cnt << (8 * (i - 4));
  }
  uint32_t ilo = plo, ihi = phi;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, ilo, o);
    const uint32_t z = __shfl_up_sync(0xffffffffu, ihi, o);
    if (lane >= o) {
      ilo += y;
      ihi += z;
    }
  }
  const uint32_t tlo = __shfl_sync(0xffffffffu, ilo, 31), thi = __shfl_sync(0xffffffffu, ihi, 31);
  const uint32_t elo = ilo - plo, ehi = ihi - phi;
  const uint32_t wtot = (tlo & 0xFFu) + ((tlo >> 8) & 0xFFu) + ((tlo >> 16) & 0xFFu) + (tlo >> 24) + (thi & 0xFFu) +
                        ((thi >> 8) & 0xFFu) + ((thi >> 16) & 0xFFu) + (thi >> 24);
  uint32_t chosen;
  uint32_t run = base + cta_warp_base(wtot, red, &chosen);
#pragma unroll
  for (int i = 0; i < V / 4; ++i) {
    const uint32_t sh = 8 * (i & 3);
    const uint32_t tot_i = ((i < 4 ? tlo : thi) >> sh) & 0xFFu;
    const uint32_t ex_i = ((i < 4 ? elo : ehi) >> sh) & 0xFFu;
    uint32_t nib = (selm >> (4 * i)) & 0xFu;
    uint32_t o = run + ex_i;
    while (nib) {
      const int cc = __ffs(nib) - 1;
      nib &= nib - 1u;
      const int p = pos_of(4 * i + cc);
      if (o < ku) out[o] = idrow ? idrow[p] : p;
      ++o;
    }
    run += tot_i;
  }
  return chosen;
}

template <int V>
__global__ void __launch_bounds__(kRThreads, 1)
topk_row_kernel(const float* __restrict__ scores, int64_t n, int64_t row_stride, const int32_t* __restrict__ row_valid,
                const int32_t* __restrict__ id_map, int64_t id_map_stride, int k, int32_t* __restrict__ idx) {
  __shared__ RSmem sm;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t t = blockIdx.x;
  const uint32_t ku = static_cast<uint32_t>(k);
  const float kNegInf = -__int_as_float(0x7f800000);
  const float kPosInf = __int_as_float(0x7f800000);
  for (int i = tid; i < kRBins; i += kRThreads) sm.hist[i] = 0u;
  sm.extra[tid] = 0u;
  if (tid == 0) sm.ccount = 0u;
  pdl_wait_inputs();
  pdl_allow_next();

  const float* row = scores + t * row_stride;
  const int32_t* idrow = id_map ? id_map + t * id_map_stride : nullptr;
  int32_t* out = idx + t * k;
  int64_t nt64 = n;
  if (row_valid) {
    const int64_t rv = row_valid[t];
    nt64 = rv < 0 ? 0 : (rv < n ? rv : n);
  }
  const int nt = static_cast<int>(nt64);
  const int wbase = warp * 32 * V;
  auto pos_of = [&](int j) { return wbase + 128 * (j >> 2) + 4 * lane + (j & 3); };

  // ---- the row in registers
  float v[V];
#pragma unroll
  for (int i = 0; i < V / 4; ++i) {
    const int p = wbase + 128 * i + 4 * lane;
    if (p + 3 < nt) {
      const float4 x = __ldg(reinterpret_cast<const float4*>(row + p));
      v[4 * i] = x.x;
      v[4 * i + 1] = x.y;
      v[4 * i + 2] = x.z;
      v[4 * i + 3] = x.w;
    } else {
#pragma unroll
      for (int c = 0; c < 4; ++c) v[4 * i + c] = p + c < nt ? __ldg(row + p + c) : kNegInf;
    }
  }
  // ---- (1) the sample's range (finite selectable values)
  const bool sok = v[0] > kNegInf && v[0] < kPosInf;
  float mn = sok ? v[0] : kPosInf, mx = sok ? v[0] : kNegInf;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  if (lane == 0) {
    sm.red[1][warp] = __float_as_uint(mn);
    sm.red[2][warp] = __float_as_uint(mx);
  }
  __syncthreads();
  mn = __uint_as_float(sm.red[1][lane]);
  mx = __uint_as_float(sm.red[2][lane]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  const float span = mx - mn;
  const float scale = static_cast<float>(kRBins) / span;
  // (a finite positive scale keeps the bin arithmetic finite and monotone)
  const float off = -mn * scale;
  const bool ranged = mx > mn && span > 0.f && isfinite(span) && isfinite(scale) && isfinite(off);
  // bin of a selectable value: round(clamp(x * scale + off, 0, 2047)) through
  // the float adder (2^23 + r holds r in its low mantissa bits); monotone in x
  auto bin_of = [&](float x) {
    const float y = fminf(fmaxf(fmaf(x, scale, off), 0.f), static_cast<float>(kRBins - 1)) + 8388608.f;
    return __float_as_uint(y) & static_cast<uint32_t>(kRBins - 1);
  };

  uint32_t selm = 0u;     // bit j: entry j is selected
  bool general = true;    // tau / take / eqtot still to be found and applied
  bool all_sel = false;   // at most k selectable entries: all of them
  uint32_t need = ku;
  uint32_t inb = 0u;      // general path, radix over registers: bit j takes part
  bool over_list = false; // general path: radix over the list
  uint32_t c = 0u;
  if (ranged) {
    // ---- (2) histogram of the range
#pragma unroll
    for (int j = 0; j < V; ++j)
      if (v[j] > kNegInf) atomicAdd(&sm.hist[bin_of(v[j])], 1u);
    __syncthreads();
    const uint32_t nsel = row_find_bin(sm, kRBins, ku, 0);
    if (nsel <= ku) {
      all_sel = true;
    } else {
      const uint32_t bstar = sm.bc[0];
      need = ku - sm.bc[1];
      c = sm.hist[bstar];
      const bool listed = c <= static_cast<uint32_t>(kRCandCap);
      // ---- (3) mark the entries above b*, list those in it
#pragma unroll
      for (int j = 0; j < V; ++j) {
        if (!(v[j] > kNegInf)) continue;
        const uint32_t b = bin_of(v[j]);
        if (b > bstar) selm |= 1u << j;
        if (b == bstar) {
          if (listed) {
            const uint32_t s = atomicAdd(&sm.ccount, 1u);
            if (s < static_cast<uint32_t>(kRCandCap)) {
              sm.cv[s] = v[j];
              sm.cp[s] = pos_of(j);
            }
          } else {
            inb |= 1u << j;
          }
        }
      }
      __syncthreads();
      if (listed && c <= static_cast<uint32_t>(kRRankMax)) {
        // rank by counting: (value descending, position ascending); the need
        // best are selected, marked in their owner's mask
        if (static_cast<uint32_t>(tid) < c) {
          const float x = sm.cv[tid];
          const int32_t px = sm.cp[tid];
          uint32_t rank = 0;
          for (uint32_t i = 0; i < c; ++i) {
            const float y = sm.cv[i];
            rank += (y > x || (y == x && sm.cp[i] < px)) ? 1u : 0u;
          }
          if (rank < need) {
            const int w = px / (32 * V), rem = px - w * 32 * V;
            const int owner = w * 32 + ((rem >> 2) & 31);
            atomicOr(&sm.extra[owner], 1u << (4 * (rem >> 7) + (rem & 3)));
          }
        }
        __syncthreads();
        selm |= sm.extra[tid];
        general = false;
      } else {
        over_list = listed;
      }
    }
  } else {
    uint32_t nl = 0;
#pragma unroll
    for (int j = 0; j < V; ++j)
      if (v[j] > kNegInf) {
        inb |= 1u << j;
        ++nl;
      }
    uint32_t nsel;
    row_warp_base(sm, warp_sum(nl), 0, &nsel);
    all_sel = nsel <= ku;
  }

  if (all_sel) {
#pragma unroll
    for (int j = 0; j < V; ++j)
      if (v[j] > kNegInf) selm |= 1u << j;
  } else if (general) {
    // ---- general path: tau by radix rounds over the list or the registers
    if (over_list) {
      row_radix(sm, need, [&](uint32_t prefix, uint32_t pmask, int sh, int nb) {
        for (uint32_t i = tid; i < c; i += kRThreads) {
          const uint32_t kk = float_key(sm.cv[i]);
          if ((kk & pmask) == prefix) atomicAdd(&sm.hist[(kk >> sh) & static_cast<uint32_t>(nb - 1)], 1u);
        }
      });
    } else {
      row_radix(sm, need, [&](uint32_t prefix, uint32_t pmask, int sh, int nb) {
#pragma unroll
        for (int j = 0; j < V; ++j) {
          const uint32_t kk = float_key(v[j]);
          if (((inb >> j) & 1u) && (kk & pmask) == prefix)
            atomicAdd(&sm.hist[(kk >> sh) & static_cast<uint32_t>(nb - 1)], 1u);
        }
      });
    }
    const float tau = sm.tau;
    const uint32_t take = sm.take, eqtot = sm.eqtot;
    // entries above tau, and of those equal to it the lowest positions
    uint32_t tk = 0u;
#pragma unroll
    for (int j = 0; j < V; ++j)
      if (v[j] == tau) tk |= 1u << j;
    if (eqtot > take) tk = cta_keep_first<V>(tk, take, sm.red[0]);   // (CTA-uniform)
    selm = tk;
#pragma unroll
    for (int j = 0; j < V; ++j)
      if (v[j] > tau) selm |= 1u << j;
  }

  // ---- (4) slots in position order
  const uint32_t chosen = cta_write_selected<V>(selm, 0u, pos_of, idrow, out, ku, sm.red[1]);
  for (uint32_t i = chosen + tid; i < ku; i += kRThreads) out[i] = -1;
}

// ---------------------------------------------------------------------------
// Rows of 8193 .. 131072 entries, few rows (topk_rowc_kernel): the algorithm
// of topk_row_kernel over a cluster of CL CTAs per row (1024 threads, V = 8 or
// 16 entries each; CTA r holds positions [r 1024V, (r+1) 1024V)), so that each
// pass over the row's registers is CL times shorter.  Every CTA takes the same
// sample (1024 evenly spaced positions of the whole row), so all agree on the
// value range without an exchange.  Two cluster barriers on the common path:
// after the histograms (each CTA sums the CL histograms through distributed
// shared memory and finds b* itself) and after the lists of b*'s entries
// (each CTA gathers the cluster's list, ranks every entry and marks its own;
// the slots before CTA r follow from every CTA's count above b* and its
// selected listed entries).  General path: three radix rounds whose
// histograms are summed the same way, then every CTA's counts above and equal
// to tau.  No CTA exits while another may still read its shared memory.
constexpr int kCMaxCL = 8;

struct alignas(16) CSmem {
  uint32_t hist[2][kRBins];   // own histograms (read by the cluster): [0] range, radix round 1; [1] rounds 0, 2
  uint32_t ghist[kRBins];     // the cluster's sum
  float cv[kRRankMax];        // own entries of b* (read by the cluster)
  int32_t cp[kRRankMax];
  float uv[kRRankMax];        // the cluster's entries of b*, in CTA order
  int32_t up[kRRankMax];
  uint32_t ur[kRRankMax];     // ... and the CTA holding each
  uint32_t extra[kRThreads];  // per thread: listed entries that are selected (bit j)
  uint32_t red[3][kRWarps];
  uint32_t bc[2];
  uint32_t meta[4];           // own counts (read by the cluster): selectable, above tau, equal to tau, listed
  uint32_t gsrc[kCMaxCL];     // per CTA: entries above b*
  uint32_t csrc[kCMaxCL];     // per CTA: listed entries selected
};

template <int V>
__global__ void __launch_bounds__(kRThreads, 1)
topk_rowc_kernel(const float* __restrict__ scores, int64_t n, int64_t row_stride, const int32_t* __restrict__ row_valid,
                 const int32_t* __restrict__ id_map, int64_t id_map_stride, int k, int32_t* __restrict__ idx) {
  __shared__ CSmem sm;
  cg::cluster_group cl = cg::this_cluster();
  const int CL = static_cast<int>(cl.num_blocks());
  const int rank = static_cast<int>(cl.block_rank());
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t t = blockIdx.y;
  const uint32_t ku = static_cast<uint32_t>(k);
  const float kNegInf = -__int_as_float(0x7f800000);
  const float kPosInf = __int_as_float(0x7f800000);
  for (int i = tid; i < kRBins; i += kRThreads) sm.hist[0][i] = 0u;
  sm.extra[tid] = 0u;
  if (tid < 4) sm.meta[tid] = 0u;
  if (tid < kCMaxCL) {
    sm.gsrc[tid] = 0u;
    sm.csrc[tid] = 0u;
  }
  pdl_wait_inputs();
  pdl_allow_next();

  const float* row = scores + t * row_stride;
  const int32_t* idrow = id_map ? id_map + t * id_map_stride : nullptr;
  int32_t* out = idx + t * k;
  int64_t nt64 = n;
  if (row_valid) {
    const int64_t rv = row_valid[t];
    nt64 = rv < 0 ? 0 : (rv < n ? rv : n);
  }
  const int nt = static_cast<int>(nt64);
  const int wbase = rank * kRThreads * V + warp * 32 * V;
  auto pos_of = [&](int j) { return wbase + 128 * (j >> 2) + 4 * lane + (j & 3); };

  float v[V];
#pragma unroll
  for (int i = 0; i < V / 4; ++i) {
    const int p = wbase + 128 * i + 4 * lane;
    if (p + 3 < nt) {
      const float4 x = __ldg(reinterpret_cast<const float4*>(row + p));
      v[4 * i] = x.x;
      v[4 * i + 1] = x.y;
      v[4 * i + 2] = x.z;
      v[4 * i + 3] = x.w;
    } else {
#pragma unroll
      for (int c = 0; c < 4; ++c) v[4 * i + c] = p + c < nt ? __ldg(row + p + c) : kNegInf;
    }
  }
  // ---- (1) the range of a sample of the whole row (the same in every CTA)
  const float smp = nt > 0 ? __ldg(row + static_cast<int64_t>(tid) * nt / kRThreads) : kNegInf;
  const bool sok = smp > kNegInf && smp < kPosInf;
  float mn = sok ? smp : kPosInf, mx = sok ? smp : kNegInf;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  if (lane == 0) {
    sm.red[1][warp] = __float_as_uint(mn);
    sm.red[2][warp] = __float_as_uint(mx);
  }
  __syncthreads();
  mn = __uint_as_float(sm.red[1][lane]);
  mx = __uint_as_float(sm.red[2][lane]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  const float span = mx - mn;
  const float scale = static_cast<float>(kRBins) / span;
  const float off = -mn * scale;
  const bool ranged = mx > mn && span > 0.f && isfinite(span) && isfinite(scale) && isfinite(off);
  auto bin_of = [&](float x) {
    const float y = fminf(fmaxf(fmaf(x, scale, off), 0.f), static_cast<float>(kRBins - 1)) + 8388608.f;
    return __float_as_uint(y) & static_cast<uint32_t>(kRBins - 1);
  };

  // ---- (2) own histogram (or, with no range, the selectable entries)
  uint32_t inb = 0u, nl = 0u;
#pragma unroll
  for (int j = 0; j < V; ++j) {
    if (!(v[j] > kNegInf)) continue;
    ++nl;
    if (ranged) atomicAdd(&sm.hist[0][bin_of(v[j])], 1u);
    else inb |= 1u << j;
  }
  nl = warp_sum(nl);
  if (lane == 0 && nl) atomicAdd(&sm.meta[0], nl);
  cl.sync();   // every CTA's histogram and selectable count are complete

  const uint32_t src_sel = lane < CL ? cl.map_shared_rank(&sm.meta[0], lane)[0] : 0u;
  const uint32_t nsel = warp_sum(src_sel);
  uint32_t selm = 0u;       // bit j: entry j is selected
  uint32_t base = 0u;       // slots before this CTA's entries
  uint32_t need = ku;
  bool general = false;
  if (nsel <= ku) {
#pragma unroll
    for (int j = 0; j < V; ++j)
      if (v[j] > kNegInf) selm |= 1u << j;
    base = warp_sum(lane < rank ? src_sel : 0u);
  } else if (ranged) {
    // the cluster's histogram: this thread's two bins of every CTA
    uint2 hs[kCMaxCL];
#pragma unroll
    for (int r = 0; r < kCMaxCL; ++r)
      hs[r] = r < CL ? reinterpret_cast<const uint2*>(cl.map_shared_rank(&sm.hist[0][0], r))[tid] : make_uint2(0u, 0u);
    uint2 g = make_uint2(0u, 0u);
#pragma unroll
    for (int r = 0; r < kCMaxCL; ++r) {
      g.x += hs[r].x;
      g.y += hs[r].y;
    }
    reinterpret_cast<uint2*>(sm.ghist)[tid] = g;
    __syncthreads();
    cta_find_bin(sm.ghist, kRBins, ku, sm.red[0], sm.bc);
    const uint32_t bstar = sm.bc[0];
    need = ku - sm.bc[1];
    const uint32_t c = sm.ghist[bstar];
    // entries above b* held by each CTA
#pragma unroll
    for (int r = 0; r < kCMaxCL; ++r) {
      if (r >= CL) break;
      uint32_t a = (2u * tid > bstar ? hs[r].x : 0u) + (2u * tid + 1u > bstar ? hs[r].y : 0u);
      a = warp_sum(a);
      if (lane == 0 && a) atomicAdd(&sm.gsrc[r], a);
    }
    if (c <= static_cast<uint32_t>(kRRankMax)) {
      // ---- (3) mark own entries above b*, list own entries in it
#pragma unroll
      for (int j = 0; j < V; ++j) {
        if (!(v[j] > kNegInf)) continue;
        const uint32_t b = bin_of(v[j]);
        if (b > bstar) selm |= 1u << j;
        if (b == bstar) {
          const uint32_t s2 = atomicAdd(&sm.meta[3], 1u);
          if (s2 < static_cast<uint32_t>(kRRankMax)) {
            sm.cv[s2] = v[j];
            sm.cp[s2] = pos_of(j);
          }
        }
      }
      cl.sync();   // every CTA's list is complete
      // the cluster's list in CTA order (warp r copies CTA r's)
      if (warp < CL) {
        const uint32_t cnt_l = lane < CL ? cl.map_shared_rank(&sm.meta[3], lane)[0] : 0u;
        uint32_t inc = cnt_l;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
          if (lane >= o) inc += y;
        }
        const uint32_t off_r = __shfl_sync(0xffffffffu, inc - cnt_l, warp);
        const uint32_t cnt_r = __shfl_sync(0xffffffffu, cnt_l, warp);
        const float* rcv = cl.map_shared_rank(&sm.cv[0], warp);
        const int32_t* rcp = cl.map_shared_rank(&sm.cp[0], warp);
        for (uint32_t i = lane; i < cnt_r && off_r + i < static_cast<uint32_t>(kRRankMax); i += 32) {
          sm.uv[off_r + i] = rcv[i];
          sm.up[off_r + i] = rcp[i];
          sm.ur[off_r + i] = static_cast<uint32_t>(warp);
        }
      }
      __syncthreads();
      // rank by counting over the cluster's list; the need best are selected
      if (static_cast<uint32_t>(tid) < c) {
        const float x = sm.uv[tid];
        const int32_t px = sm.up[tid];
        uint32_t rk = 0;
        for (uint32_t i = 0; i < c; ++i) {
          const float y = sm.uv[i];
          rk += (y > x || (y == x && sm.up[i] < px)) ? 1u : 0u;
        }
        if (rk < need) {
          const uint32_t owner_cta = sm.ur[tid];
          atomicAdd(&sm.csrc[owner_cta], 1u);
          if (owner_cta == static_cast<uint32_t>(rank)) {
            const int loc = px - rank * kRThreads * V;
            const int w = loc / (32 * V), rem = loc - w * 32 * V;
            atomicOr(&sm.extra[w * 32 + ((rem >> 2) & 31)], 1u << (4 * (rem >> 7) + (rem & 3)));
          }
        }
      }
      __syncthreads();
      selm |= sm.extra[tid];
      for (int r = 0; r < rank; ++r) base += sm.gsrc[r] + sm.csrc[r];
    } else {
      general = true;
#pragma unroll
      for (int j = 0; j < V; ++j)
        if (v[j] > kNegInf && bin_of(v[j]) == bstar) inb |= 1u << j;
    }
  } else {
    general = true;   // inb: every selectable entry
  }

  if (general) {
    // ---- general path: radix rounds over the cluster's marked entries
    uint32_t prefix = 0u, pmask = 0u, eqtot = 0u;
#pragma unroll 1
    for (int round = 0; round < 3; ++round) {
      const int sh = round == 0 ? 21 : (round == 1 ? 10 : 0);
      const int nb = round == 2 ? 1024 : 2048;
      uint32_t* hb = sm.hist[round == 1 ? 0 : 1];
      __syncthreads();
      for (int i = tid; i < nb; i += kRThreads) hb[i] = 0u;
      __syncthreads();
#pragma unroll
      for (int j = 0; j < V; ++j) {
        const uint32_t kk = float_key(v[j]);
        if (((inb >> j) & 1u) && (kk & pmask) == prefix) atomicAdd(&hb[(kk >> sh) & static_cast<uint32_t>(nb - 1)], 1u);
      }
      cl.sync();   // every CTA's round histogram is complete (and the previous one of this buffer read)
      for (int i = tid; i < nb; i += kRThreads) {
        uint32_t g = 0u;
        for (int r = 0; r < CL; ++r) g += cl.map_shared_rank(hb, r)[i];
        sm.ghist[i] = g;
      }
      __syncthreads();
      cta_find_bin(sm.ghist, nb, need, sm.red[round & 1], sm.bc);
      const uint32_t d = sm.bc[0];
      need -= sm.bc[1];
      prefix |= d << sh;
      pmask |= static_cast<uint32_t>(nb - 1) << sh;
      if (round == 2) eqtot = sm.ghist[d];
    }
    const float tau = key_to_float(prefix);
    const uint32_t take = need;
    (void)eqtot;
    uint32_t gt_l = 0u, tk = 0u;
#pragma unroll
    for (int j = 0; j < V; ++j) {
      if (v[j] > tau) selm |= 1u << j;
      if (v[j] == tau) tk |= 1u << j;
    }
    gt_l = warp_sum(__popc(selm));
    const uint32_t eq_l = warp_sum(__popc(tk));
    if (lane == 0) {
      if (gt_l) atomicAdd(&sm.meta[1], gt_l);
      if (eq_l) atomicAdd(&sm.meta[2], eq_l);
    }
    cl.sync();   // every CTA's counts above and equal to tau are complete
    const uint32_t gt_r = lane < CL ? cl.map_shared_rank(&sm.meta[1], lane)[0] : 0u;
    const uint32_t eq_r = lane < CL ? cl.map_shared_rank(&sm.meta[2], lane)[0] : 0u;
    uint32_t einc = eq_r;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, einc, o);
      if (lane >= o) einc += y;
    }
    const uint32_t ebefore = einc - eq_r;   // ties held by lower CTAs
    const uint32_t taken_r = ebefore >= take ? 0u : (take - ebefore < eq_r ? take - ebefore : eq_r);
    base = warp_sum(lane < rank ? gt_r + taken_r : 0u);
    const uint32_t my_take = __shfl_sync(0xffffffffu, taken_r, rank);
    const uint32_t my_eq = __shfl_sync(0xffffffffu, eq_r, rank);
    if (my_eq > my_take) tk = cta_keep_first<V>(tk, my_take, sm.red[0]);   // (CTA-uniform)
    selm |= tk;
  }

  // no shared memory of another CTA is read past this point
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
  // ---- (4) slots: this CTA's after the lower CTAs'
  const uint32_t mine = cta_write_selected<V>(selm, base, pos_of, idrow, out, ku, sm.red[1]);
  if (rank == CL - 1) {
    const uint32_t chosen = base + mine;   // the last CTA's slots end the row's
    for (uint32_t i = chosen + tid; i < ku; i += kRThreads) out[i] = -1;
  }
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

}  // namespace

size_t topk_smem_bytes() { return kClusterSmemBytes; }

cudaError_t launch_topk(const float* scores, int T, int64_t n, int64_t row_stride, const int32_t* row_valid,
                        const int32_t* id_map, int64_t id_map_stride, int k, int32_t* idx, cudaStream_t stream) {
  // Many rows (at least two per SM): one CTA per row, no cluster traffic.
  // Few rows: a cluster per row, so that a small batch still spreads over the
  // GPU.
  const int sms = device_sm_count();
  if (sms > 0 && static_cast<int64_t>(T) >= 2 * static_cast<int64_t>(sms) && n <= kBMaxN) {
    const size_t smem = sizeof(BSmem);
    cudaError_t e = ensure_dynamic_smem(reinterpret_cast<const void*>(topk_band_kernel), static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    return launch_pdl(topk_band_kernel, dim3(T), dim3(kBThreads), smem, stream, 0, scores, n, row_stride, row_valid,
                      id_map, id_map_stride, k, idx);
  }
  if (n > static_cast<int64_t>(kRThreads) * 8 && n <= static_cast<int64_t>(kRThreads) * 16 * kCMaxCL) {
    // a cluster per row, the row in registers: 8 entries per thread, or 16
    // when 8 would need more CTAs than there are SMs (or more than 8 per row)
    const int64_t cl8 = (n + kRThreads * 8 - 1) / (kRThreads * 8);
    const bool v8 = cl8 <= kCMaxCL && (sms <= 0 || static_cast<int64_t>(T) * cl8 <= sms);
    const int V = v8 ? 8 : 16;
    const int CL = static_cast<int>((n + static_cast<int64_t>(kRThreads) * V - 1) / (static_cast<int64_t>(kRThreads) * V));
    auto go = [&](auto kern) -> cudaError_t {
      return launch_pdl(kern, dim3(CL, T, 1), dim3(kRThreads), 0, stream, CL, scores, n, row_stride, row_valid,
                        id_map, id_map_stride, k, idx);
    };
    if (V == 8) return go(topk_rowc_kernel<8>);
    return go(topk_rowc_kernel<16>);
  }
  if (n <= static_cast<int64_t>(kRThreads) * 8) {
    // one CTA per row, the row in registers: V entries per thread
    const int V = n <= kRThreads * 4 ? 4 : 8;
    auto go = [&](auto kern) -> cudaError_t {
      return launch_pdl(kern, dim3(T), dim3(kRThreads), 0, stream, 0, scores, n, row_stride, row_valid, id_map,
                        id_map_stride, k, idx);
    };
    if (V == 4) return go(topk_row_kernel<4>);
    return go(topk_row_kernel<8>);
  }
  // longer rows: a cluster of 8, slices starting on 16-byte boundaries
  const int CL = kMaxCluster;
  int64_t slice = (n + CL - 1) / CL;
  slice = (slice + 3) / 4 * 4;
  const size_t smem = topk_smem_bytes();
  cudaError_t e = ensure_dynamic_smem(reinterpret_cast<const void*>(topk_cluster_kernel), static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  return launch_pdl(topk_cluster_kernel, dim3(CL, T, 1), dim3(kThreads), smem, stream, CL, scores, n, row_stride,
                    row_valid, id_map, id_map_stride, k, idx, slice);
}

}  // namespace misa
