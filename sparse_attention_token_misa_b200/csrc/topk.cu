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
// Rows of up to 40960 entries: one 1024-thread CTA per row keeps the whole
// row in shared memory (topk_row_kernel; value-range histogram, a position
// bitmap of the chosen entries, ascending output from its population counts).  Longer rows are split into CL
// contiguous slices, one per CTA of a cluster of CL CTAs (CL = 2..8, by row
// length; topk_cluster_kernel).  Scores become order-preserving uint32 keys,
// kept in shared memory for the whole selection, so the row is read from
// global memory exactly once.  The k-th largest key tau is found digit by
// digit (12 + 10 + 10 bits): every CTA histograms the digit over its slice
// (keys whose higher digits match the prefix found so far), the CL histograms
// are summed through distributed shared memory (each CTA owns 1/CL of the
// bins), every CTA pulls the summed histogram and finds the bin holding the
// k-th key.  A final pass writes the selected positions: each warp owns a
// contiguous chunk of its slice, warp ballots, a scan over the warps and the
// per-CTA counts exchanged across the cluster give every selected entry its
// output slot, so the output is in position order without a sort.  Keys equal to tau are taken lowest
// position first, exactly as many as needed.
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
  uint32_t counts[2];      // (above tau, equal to tau) in this CTA's slice
  uint64_t warp_tot64[kWarps];
  uint64_t block_tot64;
};
constexpr size_t kKeysOff = (sizeof(Smem) + 15) / 16 * 16;

__device__ __forceinline__ bool selectable(float v) { return v == v && v > -__int_as_float(0x7f800000); }

// key of a score, 0 for entries that can never be selected
__device__ __forceinline__ uint32_t sel_key(float v) { return selectable(v) ? float_key(v) : 0u; }

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
    uint32_t s = 0;
    for (int c = 0; c < CL; ++c) s += cl.map_shared_rank(&sm.hist[0], c)[base + i];
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
  for (int c = 0; c < CL; ++c) {
    const uint32_t* rc = cl.map_shared_rank(&sm.counts[0], c);
    const uint32_t ca = rc[0], ce = rc[1];
    if (c < rank) {
      a_before += ca;
      e_before += ce;
    }
    a_all += ca;
    e_all += ce;
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
// One CTA per row, for rows that fit in shared memory (decode rows, candidate
// lists, block scores): no cluster barriers.  Instead of bit digits (whose top
// bits put most scores of a row into a handful of exponent bins, serialising the
// shared-memory atomics) the first pass histograms the scores into 4096 equal
// value ranges between the row's min and max, a monotone map, so the threshold
// bin holds few entries.  Those candidates are collected with one atomic per
// warp and the exact threshold among them is found by counting (few) or by a
// bit-digit radix select over them (many).
constexpr int kRowThreads = 1024;
constexpr int kRowWarps = kRowThreads / 32;
constexpr int kRowBins = 4096;
constexpr int kRowMaxN = 40960;    // scores held in shared memory
constexpr int kRowCandCap = 4096;  // entries of the threshold bin kept
constexpr int kRowQuadCap = 1024;  // up to this many candidates: exact rank by counting

struct RowSmem {
  uint32_t hist[kRowBins];
  float cval[kRowCandCap];
  int32_t cpos[kRowCandCap];
  uint32_t warp_u[kRowWarps];
  float warp_f[2][kRowWarps];
  uint32_t bcast[8];
  float fcast[4];
  uint32_t ccount;
};
constexpr size_t kRowValsOff = (sizeof(RowSmem) + 15) / 16 * 16;

__device__ __forceinline__ float valid_or_neg_inf(float v) { return selectable(v) ? v : -__int_as_float(0x7f800000); }

__device__ __forceinline__ uint32_t row_sum_u32(RowSmem& sm, uint32_t x) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  if (lane == 0) sm.warp_u[warp] = x;
  __syncthreads();
  uint32_t s = 0;
  for (int i = 0; i < kRowWarps; ++i) s += sm.warp_u[i];
  __syncthreads();
  return s;
}

// bin b of hist[0, nbins) with sum(hist[b+1..]) < need <= sum(hist[b..])
__device__ __forceinline__ int row_find_bin(RowSmem& sm, int nbins, uint32_t need, uint32_t* above) {
  const int per = nbins / kRowThreads;
  const int b0 = threadIdx.x * per;
  uint32_t local = 0;
  for (int i = 0; i < per; ++i) local += sm.hist[b0 + i];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t inc = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_down_sync(0xffffffffu, inc, o);
    if (lane + o < 32) inc += y;
  }
  if (lane == 0) sm.warp_u[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    const uint32_t tw = sm.warp_u[lane];
    uint32_t ti = tw;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_down_sync(0xffffffffu, ti, o);
      if (lane + o < 32) ti += y;
    }
    sm.warp_u[lane] = ti - tw;
  }
  __syncthreads();
  const uint32_t after = sm.warp_u[warp] + inc - local;
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

// Radix select (12 + 10 + 10 key bits) of the need-th largest key among the
// entries i < cnt of `src` for which in_set(v) holds; returns its key and sets
// *gt = number of those entries with a larger key.
template <class Src, class InSet>
__device__ uint32_t row_radix_select(RowSmem& sm, Src src, int cnt, InSet in_set, uint32_t need, uint32_t* gt) {
  uint32_t prefix = 0, above = 0;
  const int shift[3] = {20, 10, 0};
  const uint32_t mask[3] = {0xfffu, 0x3ffu, 0x3ffu};
  for (int round = 0; round < 3; ++round) {
    const int nb = round == 0 ? kRowBins : 1024;
    for (int i = threadIdx.x; i < nb; i += kRowThreads) sm.hist[i] = 0;
    __syncthreads();
    for (int i = threadIdx.x; i < cnt; i += kRowThreads) {
      const float v = src(i);
      if (!in_set(v)) continue;
      const uint32_t kk = float_key(v);
      const bool match = round == 0 || (kk >> (shift[round - 1])) == prefix;
      if (match) atomicAdd(&sm.hist[(kk >> shift[round]) & mask[round]], 1u);
    }
    __syncthreads();
    uint32_t a;
    const int b = row_find_bin(sm, nb, need, &a);
    above += a;
    need -= a;
    prefix = round == 0 ? static_cast<uint32_t>(b) : ((prefix << 10) | static_cast<uint32_t>(b));
  }
  *gt = above;
  return prefix;
}

__device__ __forceinline__ float key_to_float(uint32_t kk) {
  const uint32_t u = (kk & 0x80000000u) ? (kk ^ 0x80000000u) : ~kk;
  return __uint_as_float(u);
}

__global__ void __launch_bounds__(kRowThreads, 1)
topk_row_kernel(const float* __restrict__ scores, int64_t n, int64_t row_stride, const int32_t* __restrict__ row_valid,
                const int32_t* __restrict__ id_map, int64_t id_map_stride, int k, int32_t* __restrict__ idx) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  RowSmem& sm = *reinterpret_cast<RowSmem*>(smem_raw);
  float* vals = reinterpret_cast<float*>(smem_raw + kRowValsOff);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float kNegInf = -__int_as_float(0x7f800000);
  const int64_t t = blockIdx.x;
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
  const int nwords = (nt + 31) / 32;
  uint32_t* bitmap = reinterpret_cast<uint32_t*>(vals + (nt + 3) / 4 * 4);  // 1 bit per position

  for (int i = tid; i < kRowBins; i += kRowThreads) sm.hist[i] = 0;
  if (tid == 0) sm.ccount = 0;

  // ---------------- pass A: load the row once; the value range of a sample
  // (each thread's first 16 bytes) sets the histogram's bins (values outside
  // it go to the end bins, which keeps the map monotone)
  const int nv = nt / 4;
  const float4* r4 = reinterpret_cast<const float4*>(row);
  constexpr int kPer = kRowMaxN / 4 / kRowThreads;  // float4 per thread at most (10)
  float4 f[kPer];
#pragma unroll
  for (int u = 0; u < kPer; ++u) {
    const int i = tid + u * kRowThreads;
    f[u] = i < nv ? __ldg(r4 + i) : make_float4(kNegInf, kNegInf, kNegInf, kNegInf);
  }
  float smax = kNegInf, smin = __int_as_float(0x7f800000);
  {
    const float e[4] = {valid_or_neg_inf(f[0].x), valid_or_neg_inf(f[0].y), valid_or_neg_inf(f[0].z),
                        valid_or_neg_inf(f[0].w)};
#pragma unroll
    for (int c = 0; c < 4; ++c)
      if (e[c] > kNegInf) {
        smax = fmaxf(smax, e[c]);
        smin = fminf(smin, e[c]);
      }
  }
  if (tid == 0)  // short rows: the scalar tail is part of the sample
    for (int i = 4 * nv; i < nt; ++i) {
      const float v = valid_or_neg_inf(__ldg(row + i));
      if (v > kNegInf) {
        smax = fmaxf(smax, v);
        smin = fminf(smin, v);
      }
    }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    smax = fmaxf(smax, __shfl_xor_sync(0xffffffffu, smax, o));
    smin = fminf(smin, __shfl_xor_sync(0xffffffffu, smin, o));
  }
  if (lane == 0) {
    sm.warp_f[0][warp] = smax;
    sm.warp_f[1][warp] = smin;
  }
  __syncthreads();
  smax = sm.warp_f[0][0];
  smin = sm.warp_f[1][0];
  for (int i = 1; i < kRowWarps; ++i) {
    smax = fmaxf(smax, sm.warp_f[0][i]);
    smin = fminf(smin, sm.warp_f[1][i]);
  }
  const float range = smax - smin;
  const float scale = (range > 0.f && range < __int_as_float(0x7f800000)) ? static_cast<float>(kRowBins) / range : 0.f;
  // monotone in v; any NaN intermediate (no valid sample, infinite values) maps to bin 0
  auto bin_of = [&](float v) -> int {
    const float x = (v - smin) * scale;
    return x > 0.f ? (x >= static_cast<float>(kRowBins - 1) ? kRowBins - 1 : static_cast<int>(x)) : 0;
  };
  uint32_t nvalid = 0;
#pragma unroll
  for (int u = 0; u < kPer; ++u) {
    const int i = tid + u * kRowThreads;
    if (i < nv) {
      const float4 g = make_float4(valid_or_neg_inf(f[u].x), valid_or_neg_inf(f[u].y), valid_or_neg_inf(f[u].z),
                                   valid_or_neg_inf(f[u].w));
      *reinterpret_cast<float4*>(&vals[4 * i]) = g;
      const float e[4] = {g.x, g.y, g.z, g.w};
#pragma unroll
      for (int c = 0; c < 4; ++c)
        if (e[c] > kNegInf) {
          atomicAdd(&sm.hist[bin_of(e[c])], 1u);
          ++nvalid;
        }
    }
  }
  for (int i = 4 * nv + tid; i < nt; i += kRowThreads) {
    const float v = valid_or_neg_inf(__ldg(row + i));
    vals[i] = v;
    if (v > kNegInf) {
      atomicAdd(&sm.hist[bin_of(v)], 1u);
      ++nvalid;
    }
  }
  const uint32_t total = row_sum_u32(sm, nvalid);  // (synchronises)

  // ---------------- threshold bin, then pass B: one sweep sets the bitmap of
  // every entry above the threshold bin (warp ballots, one word per step) and
  // collects the threshold bin's entries as candidates
  int b1 = -1;
  uint32_t need = 0;
  if (total > static_cast<uint32_t>(k)) {
    uint32_t gt1;
    b1 = row_find_bin(sm, kRowBins, static_cast<uint32_t>(k), &gt1);
    need = static_cast<uint32_t>(k) - gt1;
  }
  const uint32_t nb1 = b1 >= 0 ? sm.hist[b1] : 0u;
  const bool keep_cand = nb1 <= static_cast<uint32_t>(kRowCandCap);
  for (int w = warp; w < nwords; w += kRowWarps) {
    const int i = w * 32 + lane;
    const float v = i < nt ? vals[i] : kNegInf;
    const bool valid = v > kNegInf;
    const int b = valid ? bin_of(v) : -1;
    const uint32_t above = __ballot_sync(0xffffffffu, valid && b > b1);
    const uint32_t inbin = __ballot_sync(0xffffffffu, valid && b == b1);
    if (lane == 0) bitmap[w] = above;
    if (keep_cand && inbin) {
      uint32_t base = 0;
      if (lane == 0) base = atomicAdd(&sm.ccount, static_cast<uint32_t>(__popc(inbin)));
      base = __shfl_sync(0xffffffffu, base, 0);
      if ((inbin >> lane) & 1u) {
        const uint32_t slot = base + __popc(inbin & ((1u << lane) - 1u));
        sm.cval[slot] = v;
        sm.cpos[slot] = i;
      }
    }
  }
  __syncthreads();

  if (b1 >= 0) {
    // ---------------- exact threshold tau inside bin b1, and how many entries
    // equal to tau are taken (the lowest positions)
    float tau;
    uint32_t need_eq;
    if (nb1 <= static_cast<uint32_t>(kRowQuadCap)) {
      const int c = static_cast<int>(nb1);
      if (tid < c) {
        const float v = sm.cval[tid];
        uint32_t g = 0, ge = 0;
        for (int j = 0; j < c; ++j) {
          const float u = sm.cval[j];
          g += u > v ? 1u : 0u;
          ge += u >= v ? 1u : 0u;
        }
        if (g < need && need <= ge) {
          sm.fcast[0] = v;
          sm.bcast[2] = need - g;
        }
      }
      __syncthreads();
      tau = sm.fcast[0];
      need_eq = sm.bcast[2];
    } else {
      uint32_t gt, kk;
      if (keep_cand)
        kk = row_radix_select(sm, [&](int i) { return sm.cval[i]; }, static_cast<int>(nb1), [](float) { return true; },
                              need, &gt);
      else
        kk = row_radix_select(sm, [&](int i) { return vals[i]; }, nt,
                              [&](float v) { return v > kNegInf && bin_of(v) == b1; }, need, &gt);
      tau = key_to_float(kk);
      need_eq = need - gt;
    }
    // ---------------- mark the chosen entries of bin b1 in the bitmap
    if (keep_cand) {
      const int c = static_cast<int>(nb1);
      for (int x = tid; x < c; x += kRowThreads) {
        const float v = sm.cval[x];
        bool take = v > tau;
        if (!take && v == tau) {  // rank among the equal entries by position
          const int p = sm.cpos[x];
          uint32_t r = 0;
          for (int j = 0; j < c; ++j) r += (sm.cval[j] == tau && sm.cpos[j] < p) ? 1u : 0u;
          take = r < need_eq;
        }
        if (take) atomicOr(&bitmap[sm.cpos[x] >> 5], 1u << (sm.cpos[x] & 31));
      }
    } else {
      // the bin is too large to keep: sweep it in position order
      uint32_t eq_before = 0;
      for (int w0 = 0; w0 < nwords; w0 += kRowWarps) {
        const int w = w0 + warp;
        const int i = w * 32 + lane;
        const float v = (w < nwords && i < nt) ? vals[i] : kNegInf;
        const bool inb = v > kNegInf && bin_of(v) == b1;
        const bool gtt = inb && v > tau;
        const bool eqt = inb && v == tau;
        const uint32_t beq = __ballot_sync(0xffffffffu, eqt);
        if (lane == 0) sm.warp_u[warp] = __popc(beq);
        __syncthreads();
        uint32_t before_w = eq_before, tot_w = 0;
        for (int j = 0; j < kRowWarps; ++j) {
          if (j < warp) before_w += sm.warp_u[j];
          tot_w += sm.warp_u[j];
        }
        const uint32_t my_rank = before_w + __popc(beq & ((1u << lane) - 1u));
        const bool take = gtt || (eqt && my_rank < need_eq);
        const uint32_t bt = __ballot_sync(0xffffffffu, take);
        if (lane == 0 && w < nwords && bt) bitmap[w] |= bt;
        eq_before += tot_w;
        __syncthreads();
      }
    }
  } else {
    // every valid entry is chosen: the whole bitmap is "above" already (b1 = -1)
  }
  __syncthreads();

  // ---------------- output: positions of the set bits, ascending (one word
  // per thread step, block-wide prefix over the words' population counts)
  uint32_t base = 0;
  for (int w0 = 0; w0 < nwords; w0 += kRowThreads) {
    const int w = w0 + tid;
    const uint32_t bits = w < nwords ? bitmap[w] : 0u;
    const uint32_t cnt = __popc(bits);
    uint32_t inc = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += y;
    }
    if (lane == 31) sm.warp_u[warp] = inc;
    __syncthreads();
    if (warp == 0) {
      const uint32_t tw = sm.warp_u[lane];
      uint32_t ti = tw;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, ti, o);
        if (lane >= o) ti += y;
      }
      sm.warp_u[lane] = ti - tw;
      if (lane == 31) sm.bcast[3] = ti;
    }
    __syncthreads();
    uint32_t slot = base + sm.warp_u[warp] + inc - cnt;
    uint32_t b = bits;
    while (b) {
      const int bit = __ffs(b) - 1;
      b &= b - 1;
      const int pos = w * 32 + bit;
      if (slot < static_cast<uint32_t>(k)) out[slot] = idrow ? idrow[pos] : pos;
      ++slot;
    }
    base += sm.bcast[3];
    __syncthreads();
  }
  for (uint32_t i = base + tid; i < static_cast<uint32_t>(k); i += kRowThreads) out[i] = -1;
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
  if (n <= kRowMaxN) {
    // the row's values, then a bitmap of n bits
    auto row_smem = [](int64_t m) { return kRowValsOff + static_cast<size_t>((m + 3) / 4 * 4) * 4 + ((m + 31) / 32) * 4; };
    const size_t smem = row_smem(n);
    cudaError_t e = ensure_dynamic_smem(reinterpret_cast<const void*>(topk_row_kernel), static_cast<int>(row_smem(kRowMaxN)));
    if (e != cudaSuccess) return e;
    return launch_pdl(topk_row_kernel, dim3(T), dim3(kRowThreads), smem, stream, 0, scores, n, row_stride, row_valid,
                      id_map, id_map_stride, k, idx);
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
