// Per-row top-k of fp32 scores by radix select, one thread-block cluster per row.
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
// Rows of up to 65536 entries (topk_range_kernel): a cluster of up to 8 CTAs
// per row, the row's entries held in registers, a value-range histogram whose
// threshold bin is gathered across the cluster; described above the kernel.
//
// Longer rows (topk_cluster_kernel) are split into CL = 8 contiguous slices,
// one per CTA of a cluster.  Scores become order-preserving uint32 keys
// (re-read from global memory when a slice does not fit in shared memory).
// The k-th largest key tau is found digit by digit (12 + 10 + 10 bits): every
// CTA histograms the digit over its slice (keys whose higher digits match the
// prefix found so far), the CL histograms are summed through distributed
// shared memory (each CTA owns 1/CL of the bins), every CTA pulls the summed
// histogram and finds the bin holding the k-th key.  A final pass writes the
// selected positions: each warp owns a contiguous chunk of its slice, warp
// ballots, a scan over the warps and the per-CTA counts exchanged across the
// cluster give every selected entry its output slot, so the output is in
// position order without a sort.
//
// In both kernels keys equal to tau are taken lowest position first, exactly
// as many as needed.
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
constexpr int kSliceCap = 16384;  // keys kept in shared memory per CTA

struct Smem {
  uint32_t hist[kBins1];   // local histogram, then the pulled cluster histogram
  uint32_t own[kBins1];    // this CTA's share of the summed histogram
  uint32_t warp_tot[kWarps];
  uint32_t bcast[4];
  alignas(8) uint32_t counts[2];  // (above tau, equal to tau) in this CTA's slice
  uint64_t warp_tot64[kWarps];
  uint64_t block_tot64;
};
constexpr size_t kKeysOff = (sizeof(Smem) + 15) / 16 * 16;

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

template <bool kKeysInSmem>
__global__ void __launch_bounds__(kThreads, 2)
topk_cluster_kernel(const float* __restrict__ scores, int64_t n, int64_t row_stride, const int32_t* __restrict__ row_valid,
                    const int32_t* __restrict__ id_map, int64_t id_map_stride, int k, int32_t* __restrict__ idx,
                    int64_t slice_len) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>(smem_raw);
  uint32_t* keys = reinterpret_cast<uint32_t*>(smem_raw + kKeysOff);

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

  auto key_at = [&](int i) -> uint32_t {
    if constexpr (kKeysInSmem) return keys[i];
    else return sel_key(__ldg(row + s0 + i));
  };

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
          if constexpr (kKeysInSmem) *reinterpret_cast<uint4*>(&keys[4 * i]) = make_uint4(kk[0], kk[1], kk[2], kk[3]);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            if (kk[e]) atomicAdd(&sm.hist[kk[e] >> 20], 1u);
        }
      }
    }
    for (int i = 4 * nv + tid; i < len; i += kThreads) {
      const uint32_t kk = sel_key(__ldg(row + s0 + i));
      if constexpr (kKeysInSmem) keys[i] = kk;
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

// ---------------------------------------------------------------------------
// Rows of up to 8 x 512 x 16 entries: a cluster of CL <= 8 CTAs of 512
// threads per row, each thread holding V contiguous entries of the row in
// registers (V = 8 or 16 by row length).  Instead of bit digits (whose top
// bits put most scores of a row into a few exponent bins) the histogram splits
// the value range of a fixed sample of the row (the same 512 entries in every
// CTA, so every CTA derives the same bins) into 1024 equal ranges; the map is
// monotone, values outside the sample's range go to the end bins.  The path
// is a short chain of dependent steps, each a cluster barrier followed by
// small rounds of distributed shared memory reads (they are slow; bytes are
// kept few):
//   (1) every CTA sums the CL histograms' 32 super-bin totals, finds the
//       super-bin holding the k-th entry, then sums its 32 bins (a second
//       read round) and finds the threshold bin;
//   (2) every CTA reads the counts above the threshold bin and the threshold
//       bin's entries (few) of every slice, finds the exact threshold among
//       them by counting, and so knows how many entries above and equal to it
//       each slice holds: the output slots follow from a scan.
// A threshold bin with more entries than one read round takes is gathered in
// a second round (radix select over the gathered entries when they are many);
// one too full to gather (massive ties, a sample range spoilt by outliers)
// falls back to a cluster-wide bit-digit radix select inside it.
constexpr int kXThreads = 512;
constexpr int kXWarps = kXThreads / 32;
constexpr int kXBins = 2048;          // histogram array (fallback digits use all of it)
constexpr int kXFastBins = 1024;      // value-range bins: 2 per thread
constexpr int kXSup = kXBins / 32;
constexpr int kXFastCand = kXThreads / kMaxCluster;  // threshold-bin entries per slice read in one round
constexpr int kXCandCap = 512;        // threshold-bin entries kept per CTA
constexpr int kXMergeCap = 2048;      // and over the cluster
#ifndef MISA_TOPK_RANGE_CLUSTER
#define MISA_TOPK_RANGE_CLUSTER 8
#endif
constexpr int kXRangeCluster = MISA_TOPK_RANGE_CLUSTER;  // CTAs per row at most

struct XSmem {
  uint32_t hist[kXBins];     // this CTA's histogram (read by the cluster)
  uint32_t sup[kXSup];       // fallback: its super-bin totals (read by the cluster)
  uint32_t meta[4];          // valid entries, entries above the threshold bin, threshold-bin entries (read by the cluster)
  uint32_t cnt2[2];          // fallback: entries above / equal to tau (read by the cluster)
  uint32_t gsup[kXSup];      // super-bin totals summed over the cluster
  uint32_t gbin[32];
  uint32_t bc[8];
  float fbc;
  uint32_t rv[kMaxCluster], ra[kMaxCluster], rc[kMaxCluster];
  uint32_t at[kMaxCluster], et[kMaxCluster];
  float wmin[kXWarps], wmax[kXWarps];
  uint64_t wscan[kXWarps];
  union {
    struct {
      float cval[kXCandCap];     // this CTA's threshold-bin entries (read by the cluster)
      float fval[kXThreads];     // first kXFastCand entries of every slice, [rank][i]
      float mval[kXMergeCap];    // the cluster's threshold-bin entries, by rank
      uint8_t mrank[kXMergeCap];
    } c;
    struct {
      uint32_t h[kXBins];        // fallback digit histogram, second buffer (read by the cluster)
      uint32_t s[kXSup];
    } r;
  } u;
};

__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.aligned;" ::: "memory"); }

// One warp: among tot[0, cnt) (cnt <= 128) the index i with
// above(i) < need <= above(i) + tot[i], above(i) = sum of tot[i+1 .. cnt);
// out[0] = i, out[1] = above(i).
__device__ __forceinline__ void warp_suffix_find(const uint32_t* tot, int cnt, uint32_t need, uint32_t* out) {
  const int lane = threadIdx.x & 31;
  const int per = (cnt + 31) / 32;
  const int b0 = lane * per;
  uint32_t local = 0;
  for (int i = 0; i < per; ++i)
    if (b0 + i < cnt) local += tot[b0 + i];
  uint32_t inc = local;  // sum over lanes >= this one
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_down_sync(0xffffffffu, inc, o);
    if (lane + o < 32) inc += y;
  }
  const uint32_t after = inc - local;
  if (after < need && need <= inc) {
    uint32_t acc = after;
    for (int i = per - 1; i >= 0; --i) {
      if (b0 + i >= cnt) continue;
      const uint32_t c = tot[b0 + i];
      if (acc + c >= need) {
        out[0] = static_cast<uint32_t>(b0 + i);
        out[1] = acc;
        break;
      }
      acc += c;
    }
  }
}

// Super-bin totals of a histogram of nbins (a multiple of 128, <= 2048): each
// thread adds 4 bins, 8 lanes make one super-bin of 32.
__device__ __forceinline__ void make_supers(const uint32_t* h, uint32_t* sup, int nbins) {
  const int base = threadIdx.x * 4;
  if (base < nbins) {  // whole warps
    const uint4 x = *reinterpret_cast<const uint4*>(h + base);
    uint32_t s = x.x + x.y + x.z + x.w;
    s += __shfl_xor_sync(0xffffffffu, s, 1);
    s += __shfl_xor_sync(0xffffffffu, s, 2);
    s += __shfl_xor_sync(0xffffffffu, s, 4);
    if ((threadIdx.x & 7) == 0) sup[base / 32] = s;
  }
}

// The bin holding the need-th largest entry of the histogram summed over nsrc
// sources (hist_of(r), sup_of(r): source r's bins and super-bin totals, all
// complete); *above = entries in higher bins.  Every thread of the CTA calls.
template <class HistOf, class SupOf>
__device__ int two_level_find(XSmem& sm, int nsrc, HistOf hist_of, SupOf sup_of, int nsup, uint32_t need,
                              uint32_t* above) {
  const int tid = threadIdx.x;
  for (int i = tid; i < nsup; i += kXThreads) sm.gsup[i] = 0;
  if (tid < 32) sm.gbin[tid] = 0;
  __syncthreads();
  for (int i = tid; i < nsup * nsrc; i += kXThreads) {
    const int s = i % nsup, r = i / nsup;
    atomicAdd(&sm.gsup[s], sup_of(r)[s]);
  }
  __syncthreads();
  if (tid < 32) warp_suffix_find(sm.gsup, nsup, need, sm.bc);
  __syncthreads();
  // (the index is in range by construction; the clamps only keep a wrong
  // count from addressing outside the arrays)
  const int S = sm.bc[0] < static_cast<uint32_t>(nsup) ? static_cast<int>(sm.bc[0]) : nsup - 1;
  const uint32_t above_s = sm.bc[1];
  for (int i = tid; i < 32 * nsrc; i += kXThreads) {
    const int j = i & 31, r = i >> 5;
    atomicAdd(&sm.gbin[j], hist_of(r)[S * 32 + j]);
  }
  __syncthreads();
  if (tid < 32) warp_suffix_find(sm.gbin, 32, need - above_s, sm.bc + 2);
  __syncthreads();
  *above = above_s + sm.bc[3];
  return S * 32 + static_cast<int>(sm.bc[2] & 31u);
}

// Bit digits of a key for the radix rounds: 11, 11, 10 bits from the top.
__device__ __forceinline__ int digit_shift(int round) { return round == 0 ? 21 : (round == 1 ? 10 : 0); }
__device__ __forceinline__ int digit_bins(int round) { return round == 2 ? 1024 : 2048; }

__device__ __forceinline__ float key_to_float(uint32_t kk) {
  const uint32_t u = (kk & 0x80000000u) ? (kk ^ 0x80000000u) : ~kk;
  return __uint_as_float(u);
}

template <int V>
__global__ void __launch_bounds__(kXThreads, 2)
topk_range_kernel(const float* __restrict__ scores, int64_t n, int64_t row_stride, const int32_t* __restrict__ row_valid,
                  const int32_t* __restrict__ id_map, int64_t id_map_stride, int k, int32_t* __restrict__ idx) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  XSmem& sm = *reinterpret_cast<XSmem*>(smem_raw);
  cg::cluster_group cl = cg::this_cluster();
  const int CL = static_cast<int>(cl.num_blocks());
  const int rank = static_cast<int>(cl.block_rank());
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t t = blockIdx.y;
  constexpr int kSlice = kXThreads * V;
  const float kNegInf = -__int_as_float(0x7f800000);
  const float kPosInf = __int_as_float(0x7f800000);
  const uint32_t ku = static_cast<uint32_t>(k);

  for (int i = tid; i < kXFastBins; i += kXThreads) sm.hist[i] = 0;
  if (tid < 4) sm.meta[tid] = 0;
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
  const int s0 = rank * kSlice < nt ? rank * kSlice : nt;
  const int s1 = s0 + kSlice < nt ? s0 + kSlice : nt;
  const int p0 = s0 + tid * V;  // this thread's entries: positions [p0, p0 + V) of the row

  // ---------------- load (the slice start and p0 are multiples of 4 entries)
  float v[V];
#pragma unroll
  for (int j = 0; j < V; j += 4) {
    const int p = p0 + j;
    if (p + 3 < s1) {
      const float4 f = __ldg(reinterpret_cast<const float4*>(row + p));
      v[j] = f.x;
      v[j + 1] = f.y;
      v[j + 2] = f.z;
      v[j + 3] = f.w;
    } else {
#pragma unroll
      for (int c = 0; c < 4; ++c) v[j + c] = p + c < s1 ? __ldg(row + p + c) : kNegInf;
    }
  }
  float smp = nt > 0 ? __ldg(row + static_cast<int64_t>(tid) * nt / kXThreads) : kNegInf;
  smp = valid_or_neg_inf(smp);
  float mx = smp, mn = smp > kNegInf ? smp : kPosInf;
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
  for (int i = 1; i < kXWarps; ++i) {
    mx = fmaxf(mx, sm.wmax[i]);
    mn = fminf(mn, sm.wmin[i]);
  }
  const float range = mx - mn;
  const float scale = (range > 0.f && range < kPosInf) ? static_cast<float>(kXFastBins) / range : 0.f;
  // monotone in x; a NaN intermediate (no valid sample, infinite entries) maps to bin 0
  auto bin_of = [&](float x) -> int {
    const float y = __fmul_rn(__fsub_rn(x, mn), scale);
    return y > 0.f ? (y >= static_cast<float>(kXFastBins - 1) ? kXFastBins - 1 : static_cast<int>(y)) : 0;
  };

  // ---------------- value-range histogram of the slice
  uint32_t nval = 0;
#pragma unroll
  for (int j = 0; j < V; ++j) {
    v[j] = valid_or_neg_inf(v[j]);
    if (v[j] > kNegInf) {
      atomicAdd(&sm.hist[bin_of(v[j])], 1u);
      ++nval;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) nval += __shfl_xor_sync(0xffffffffu, nval, o);
  if (lane == 0 && nval) atomicAdd(&sm.meta[0], nval);
  __syncthreads();
  make_supers(sm.hist, sm.sup, kXFastBins);
  __syncthreads();
  cl.sync();  // (1) every CTA's histogram, super-bin totals and valid count are complete

  // ---------------- the threshold bin, from the CL histograms in two read
  // rounds of 32 x CL words each: super-bin totals, then the 32 bins of the
  // super-bin holding the k-th entry.  Thread (s, r) = (tid / 8, tid % 8)
  // reads item s of source (r + rank) mod CL (the CTAs start on different
  // SMs); 8 lanes add their sources.
  const int fs = tid >> 3, fr = tid & 7;
  const int fsrc = fr + rank < CL ? fr + rank : fr + rank - CL;
  if (tid >= 32 * kMaxCluster && tid < 32 * kMaxCluster + CL)
    sm.rv[tid - 32 * kMaxCluster] = cl.map_shared_rank(&sm.meta[0], tid - 32 * kMaxCluster)[0];
  if (tid < 32 * kMaxCluster) {
    uint32_t x = fr < CL ? cl.map_shared_rank(&sm.sup[0], fsrc)[fs] : 0u;
    x += __shfl_xor_sync(0xffffffffu, x, 1);
    x += __shfl_xor_sync(0xffffffffu, x, 2);
    x += __shfl_xor_sync(0xffffffffu, x, 4);
    if (fr == 0) sm.gsup[fs] = x;
  }
  __syncthreads();
  if (warp == 0) {
    uint32_t x = sm.gsup[lane];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    if (lane == 0) sm.bc[3] = x;  // valid entries of the row
    if (x > ku) warp_suffix_find(sm.gsup, 32, ku, sm.bc);
  }
  __syncthreads();
  const uint32_t total = sm.bc[3];

  float tau = kNegInf;  // selected: entries above tau, and the first need_eq entries equal to it
  uint32_t need_eq = 0;
  if (total <= ku) {
    if (tid < CL) {
      sm.at[tid] = sm.rv[tid];
      sm.et[tid] = 0;
    }
  } else {
    const int S = static_cast<int>(sm.bc[0] & 31u);
    const uint32_t above_s = sm.bc[1];
    if (tid < 32 * kMaxCluster) {
      uint32_t x = fr < CL ? cl.map_shared_rank(&sm.hist[0], fsrc)[S * 32 + fs] : 0u;
      x += __shfl_xor_sync(0xffffffffu, x, 1);
      x += __shfl_xor_sync(0xffffffffu, x, 2);
      x += __shfl_xor_sync(0xffffffffu, x, 4);
      if (fr == 0) sm.gbin[fs] = x;
    }
    __syncthreads();
    if (warp == 0) warp_suffix_find(sm.gbin, 32, ku - above_s, sm.bc + 4);
    __syncthreads();
    const int bstar = S * 32 + static_cast<int>(sm.bc[4] & 31u);
    const uint32_t above_b = above_s + sm.bc[5];
    const uint32_t need = ku - above_b;
    // entries above the threshold bin, and the threshold bin's entries
    uint32_t a = 0;
#pragma unroll
    for (int j = 0; j < V; ++j) {
      if (v[j] > kNegInf) {
        const int b = bin_of(v[j]);
        a += b > bstar ? 1u : 0u;
        if (b == bstar) {
          const uint32_t slot = atomicAdd(&sm.meta[2], 1u);
          if (slot < static_cast<uint32_t>(kXCandCap)) sm.u.c.cval[slot] = v[j];
        }
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
    if (lane == 0 && a) atomicAdd(&sm.meta[1], a);
    __syncthreads();
    cl.sync();  // (2) every CTA's counts and threshold-bin entries are complete
    {
      // one read round: slice r's counts and its first kXFastCand entries
      // (thread group j of CTA c reads slice (j + c) mod CL: the CTAs start on
      // different slices)
      const int j = tid / kXFastCand, i = tid - j * kXFastCand;
      if (j < CL) {
        const int r = j + rank < CL ? j + rank : j + rank - CL;
        const uint32_t* m = cl.map_shared_rank(&sm.meta[0], r);
        const float x = cl.map_shared_rank(&sm.u.c.cval[0], r)[i];
        if (i == 0) {
          sm.ra[r] = m[1];
          sm.rc[r] = m[2];
        }
        sm.u.c.fval[r * kXFastCand + i] = x;
      }
    }
    __syncthreads();
    uint32_t ctot = 0, cmax = 0;
#pragma unroll
    for (int r = 0; r < kMaxCluster; ++r) {
      const uint32_t c = r < CL ? sm.rc[r] : 0u;
      ctot += c;
      cmax = c > cmax ? c : cmax;
    }
    const bool overflow = cmax > static_cast<uint32_t>(kXCandCap) || ctot > static_cast<uint32_t>(kXMergeCap);
    if (cmax <= static_cast<uint32_t>(kXFastCand)) {
      // compact the entries read in the round above
      const int r = tid / kXFastCand, i = tid - r * kXFastCand;
      if (r < CL && static_cast<uint32_t>(i) < sm.rc[r]) {
        uint32_t off = 0;
        for (int r2 = 0; r2 < r; ++r2) off += sm.rc[r2];
        sm.u.c.mval[off + i] = sm.u.c.fval[tid];
        sm.u.c.mrank[off + i] = static_cast<uint8_t>(r);
      }
      __syncthreads();
    } else if (!overflow) {
      // a second read round for the rest of the threshold bin
      for (int i = tid; i < static_cast<int>(ctot); i += kXThreads) {
        int r = 0;
        uint32_t off = 0;
        while (off + sm.rc[r] <= static_cast<uint32_t>(i)) off += sm.rc[r++];
        sm.u.c.mval[i] = cl.map_shared_rank(&sm.u.c.cval[0], r)[i - off];
        sm.u.c.mrank[i] = static_cast<uint8_t>(r);
      }
      __syncthreads();
    }
    if (!overflow) {
      if (ctot <= static_cast<uint32_t>(kXThreads)) {
        // exact rank by counting
        if (tid < static_cast<int>(ctot)) {
          const float x = sm.u.c.mval[tid];
          uint32_t g = 0, ge = 0;
#pragma unroll 4
          for (int j = 0; j < static_cast<int>(ctot); ++j) {
            const float y = sm.u.c.mval[j];
            g += y > x ? 1u : 0u;
            ge += y >= x ? 1u : 0u;
          }
          if (g < need && need <= ge) {
            sm.fbc = x;
            sm.bc[2] = need - g;
          }
        }
        __syncthreads();
        tau = sm.fbc;
        need_eq = sm.bc[2];
      } else {
        // bit-digit radix select over the gathered entries (local; the
        // histogram arrays are no longer read by the cluster after (2))
        uint32_t prefix = 0, nd = need;
        for (int round = 0; round < 3; ++round) {
          const int sh = digit_shift(round), nb = digit_bins(round);
          for (int i = tid; i < nb; i += kXThreads) sm.hist[i] = 0;
          __syncthreads();
          for (int i = tid; i < static_cast<int>(ctot); i += kXThreads) {
            const uint32_t kk = float_key(sm.u.c.mval[i]);
            if (round == 0 || (kk >> digit_shift(round - 1)) == prefix) atomicAdd(&sm.hist[(kk >> sh) & (nb - 1)], 1u);
          }
          __syncthreads();
          make_supers(sm.hist, sm.sup, nb);
          __syncthreads();
          uint32_t ab;
          const int b = two_level_find(
              sm, 1, [&](int) { return &sm.hist[0]; }, [&](int) { return &sm.sup[0]; }, nb / 32, nd, &ab);
          nd -= ab;
          prefix = round == 0 ? static_cast<uint32_t>(b) : ((prefix << (round == 1 ? 11 : 10)) | static_cast<uint32_t>(b));
        }
        tau = key_to_float(prefix);
        need_eq = nd;
      }
      // entries above / equal to tau in every slice
      if (tid < CL) {
        sm.at[tid] = sm.ra[tid];
        sm.et[tid] = 0;
      }
      __syncthreads();
      for (int i = tid; i < static_cast<int>(ctot); i += kXThreads) {
        const float x = sm.u.c.mval[i];
        if (x > tau) atomicAdd(&sm.at[sm.u.c.mrank[i]], 1u);
        else if (x == tau) atomicAdd(&sm.et[sm.u.c.mrank[i]], 1u);
      }
    } else {
      // ---------------- fallback: cluster-wide radix select inside bin bstar.
      // Digit histograms alternate between two buffers, so a CTA never
      // overwrites one that another CTA may still be reading.
      uint32_t prefix = 0, nd = need;
      for (int round = 0; round < 3; ++round) {
        uint32_t* H = (round & 1) ? sm.u.r.h : sm.hist;
        uint32_t* S = (round & 1) ? sm.u.r.s : sm.sup;
        const int sh = digit_shift(round), nb = digit_bins(round);
        for (int i = tid; i < nb; i += kXThreads) H[i] = 0;
        __syncthreads();
#pragma unroll
        for (int j = 0; j < V; ++j) {
          if (v[j] > kNegInf && bin_of(v[j]) == bstar) {
            const uint32_t kk = float_key(v[j]);
            if (round == 0 || (kk >> digit_shift(round - 1)) == prefix) atomicAdd(&H[(kk >> sh) & (nb - 1)], 1u);
          }
        }
        __syncthreads();
        make_supers(H, S, nb);
        __syncthreads();
        cl.sync();
        uint32_t ab;
        const int b = two_level_find(
            sm, CL, [&](int r) { return cl.map_shared_rank(H, r); }, [&](int r) { return cl.map_shared_rank(S, r); },
            nb / 32, nd, &ab);
        nd -= ab;
        prefix = round == 0 ? static_cast<uint32_t>(b) : ((prefix << (round == 1 ? 11 : 10)) | static_cast<uint32_t>(b));
      }
      tau = key_to_float(prefix);
      need_eq = nd;
      uint32_t ac = 0, ec = 0;
#pragma unroll
      for (int j = 0; j < V; ++j) {
        ac += v[j] > tau ? 1u : 0u;
        ec += (v[j] > kNegInf && v[j] == tau) ? 1u : 0u;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        ac += __shfl_xor_sync(0xffffffffu, ac, o);
        ec += __shfl_xor_sync(0xffffffffu, ec, o);
      }
      if (tid < 2) sm.cnt2[tid] = 0;
      __syncthreads();
      if (lane == 0) {
        atomicAdd(&sm.cnt2[0], ac);
        atomicAdd(&sm.cnt2[1], ec);
      }
      __syncthreads();
      cl.sync();
      if (tid < CL) {
        const uint32_t* c2 = cl.map_shared_rank(&sm.cnt2[0], tid);
        sm.at[tid] = c2[0];
        sm.et[tid] = c2[1];
      }
    }
  }
  __syncthreads();
  // every value read from another CTA's shared memory has arrived: it may exit
  // once all CTAs are here
  cluster_arrive_relaxed();

  // ---------------- output slots: entries above tau before this one, plus the
  // equal entries before it (at most need_eq of them)
  uint32_t a_before = 0, e_before = 0, a_all = 0, e_all = 0;
#pragma unroll
  for (int r = 0; r < kMaxCluster; ++r) {
    const uint32_t ar = r < CL ? sm.at[r] : 0u, er = r < CL ? sm.et[r] : 0u;
    a_before += r < rank ? ar : 0u;
    e_before += r < rank ? er : 0u;
    a_all += ar;
    e_all += er;
  }
  uint32_t a_t = 0, e_t = 0;
#pragma unroll
  for (int j = 0; j < V; ++j) {
    a_t += v[j] > tau ? 1u : 0u;
    e_t += (v[j] > kNegInf && v[j] == tau) ? 1u : 0u;
  }
  uint64_t x = static_cast<uint64_t>(a_t) | (static_cast<uint64_t>(e_t) << 32);
  uint64_t incl = x;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint64_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) sm.wscan[warp] = incl;
  __syncthreads();
  uint64_t wbase = 0;
  for (int i = 0; i < warp; ++i) wbase += sm.wscan[i];
  const uint64_t excl = wbase + incl - x;
  uint32_t A = a_before + static_cast<uint32_t>(excl & 0xffffffffull);
  uint32_t E = e_before + static_cast<uint32_t>(excl >> 32);
#pragma unroll
  for (int j = 0; j < V; ++j) {
    const float y = v[j];
    if (y > tau) {
      const uint32_t slot = A + (E < need_eq ? E : need_eq);
      if (slot < ku) out[slot] = idrow ? idrow[p0 + j] : p0 + j;
      ++A;
    } else if (y > kNegInf && y == tau) {
      if (E < need_eq && A + E < ku) out[A + E] = idrow ? idrow[p0 + j] : p0 + j;
      ++E;
    }
  }
  if (rank == CL - 1) {
    const uint32_t chosen = a_all + (e_all < need_eq ? e_all : need_eq);
    for (uint32_t i = chosen + tid; i < ku; i += kXThreads) out[i] = -1;
  }
  cluster_wait();  // no CTA exits while another may still read its shared memory
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
#define MISA_BAND_UNROLL 2
#endif
constexpr int kBUnroll = MISA_BAND_UNROLL;  // steps whose loads are in flight together per warp

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
  float wmin[kBWarps], wmax[kBWarps];
  uint32_t bc[8];
  float fbc[2];
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
// n_keys keys produced by key_at(i) (0 = not a candidate); returns its key and
// sets *gt to the number of larger keys.  All threads.
template <class KeyAt>
__device__ uint32_t band_radix(BSmem& sm, int n_keys, KeyAt key_at, uint32_t need, uint32_t* gt) {
  const int tid = threadIdx.x;
  uint32_t prefix = 0, above = 0;
  for (int round = 0; round < 3; ++round) {
    const int sh = round == 0 ? 20 : (round == 1 ? 10 : 0);
    const int nb = round == 0 ? 4096 : 1024;
    for (int i = tid; i < nb; i += kBThreads) sm.hist[i] = 0;
    __syncthreads();
    for (int i = tid; i < n_keys; i += kBThreads) {
      const uint32_t kk = key_at(i);
      if (kk == 0u) continue;
      const bool match = round == 0 || (kk >> (round == 1 ? 20 : 10)) == prefix;
      if (match) atomicAdd(&sm.hist[(kk >> sh) & static_cast<uint32_t>(nb - 1)], 1u);
    }
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
  const uint32_t lt = (1u << lane) - 1u;

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

  // ---------------- pass 1 (the only read of the row on the common path)
  uint32_t a_w = 0, c_w = 0;  // (warp-uniform) entries above hi, band entries seen
  float* wcval = sm.cval + warp * kBWarpCap;
  int32_t* wcpos = sm.cpos + warp * kBWarpCap;
  for (int s0 = warp; s0 < nsteps; s0 += kBWarps * kBUnroll) {
    float xs[kBUnroll][4];
#pragma unroll
    for (int u = 0; u < kBUnroll; ++u) load_step(128 * (s0 + kBWarps * u), xs[u]);
#pragma unroll
    for (int u = 0; u < kBUnroll; ++u) {
      const int st = s0 + kBWarps * u;
      if (st >= nsteps) break;
      const int base = 128 * st;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const float x = xs[u][c];
        const bool above = x > hi_v;                  // false for NaN
        const bool band = !above && x >= lo_v;        // false for NaN and -inf
        const uint32_t am = __ballot_sync(0xffffffffu, above);
        const uint32_t bm = __ballot_sync(0xffffffffu, band);
        if (lane == 0) sm.gt[(base >> 5) + c] = am;
        a_w += __popc(am);
        if (band) {
          const uint32_t sl = c_w + __popc(bm & lt);
          if (sl < static_cast<uint32_t>(kBWarpCap)) {
            wcval[sl] = x;
            wcpos[sl] = base + 32 * c + lane;
          }
        }
        c_w += __popc(bm);
      }
    }
  }
  if (lane == 0) {
    sm.wa[warp] = a_w;
    sm.wc[warp] = c_w;
  }
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
    uint32_t gt;
    const uint32_t kk = band_radix(
        sm, kBCandCap,
        [&](int i) {
          return (i % kBWarpCap) < static_cast<int>(sm.wc[i / kBWarpCap]) ? float_key(sm.cval[i]) : 0u;
        },
        ku - A, &gt);
    tau = key_to_float(kk);
    need_eq = ku - A - gt;
    for (int i = tid; i < kBCandCap; i += kBThreads) {
      if ((i % kBWarpCap) >= static_cast<int>(sm.wc[i / kBWarpCap])) continue;
      const float x = sm.cval[i];
      const int p = sm.cpos[i];
      if (x > tau) atomicOr(&sm.gt[p >> 5], 1u << (p & 31));
      else if (x == tau) atomicOr(&sm.eq[p >> 5], 1u << (p & 31));
    }
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

int pick_cluster(int64_t n) {
  int cl = 1;
  while (cl < kMaxCluster && static_cast<int64_t>(cl) * kSliceCap < n) cl <<= 1;
  return cl;
}

}  // namespace

size_t topk_smem_bytes() { return kKeysOff + static_cast<size_t>(kSliceCap) * 4; }

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
  if (n <= static_cast<int64_t>(kXRangeCluster) * kXThreads * 16) {
    // smallest V with ceil(n / (512 V)) <= kXRangeCluster CTAs per row
    const int V = n <= static_cast<int64_t>(kXRangeCluster) * kXThreads * 8 ? 8 : 16;
    const int64_t slice = static_cast<int64_t>(kXThreads) * V;
    const int CL = static_cast<int>((n + slice - 1) / slice);
    const size_t smem = sizeof(XSmem);
    auto go = [&](auto kern) -> cudaError_t {
      cudaError_t e = ensure_dynamic_smem(reinterpret_cast<const void*>(kern), static_cast<int>(smem));
      if (e != cudaSuccess) return e;
      return launch_pdl(kern, dim3(CL, T, 1), dim3(kXThreads), smem, stream, CL, scores, n, row_stride, row_valid,
                        id_map, id_map_stride, k, idx);
    };
    if (V == 8) return go(topk_range_kernel<8>);
    return go(topk_range_kernel<16>);
  }
  const int CL = pick_cluster(n);
  int64_t slice = (n + CL - 1) / CL;
  slice = (slice + 3) / 4 * 4;  // slices start on 16-byte boundaries
  const bool in_smem = slice <= kSliceCap;
  const size_t smem = in_smem ? kKeysOff + static_cast<size_t>(slice) * 4 : kKeysOff;
  const void* fn = in_smem ? reinterpret_cast<const void*>(topk_cluster_kernel<true>)
                           : reinterpret_cast<const void*>(topk_cluster_kernel<false>);
  cudaError_t e = ensure_dynamic_smem(fn, static_cast<int>(topk_smem_bytes()));
  if (e != cudaSuccess) return e;

  if (in_smem)
    return launch_pdl(topk_cluster_kernel<true>, dim3(CL, T, 1), dim3(kThreads), smem, stream, CL, scores, n,
                      row_stride, row_valid, id_map, id_map_stride, k, idx, slice);
  return launch_pdl(topk_cluster_kernel<false>, dim3(CL, T, 1), dim3(kThreads), smem, stream, CL, scores, n,
                    row_stride, row_valid, id_map, id_map_stride, k, idx, slice);
}

}  // namespace misa
