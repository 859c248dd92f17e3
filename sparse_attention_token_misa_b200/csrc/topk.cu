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
// row's keys in shared memory (topk_row_kernel).  Longer rows are split into CL
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
    if (is_a) {
      out[my_a + (my_e < need_eq ? my_e : need_eq)] = idrow ? idrow[s0 + i] : static_cast<int32_t>(s0 + i);
    } else if (is_e && my_e < need_eq) {
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
// One CTA per row, for rows whose keys fit in shared memory (decode rows,
// candidate lists, block scores): no cluster barriers at all.
constexpr int kRowThreads = 1024;
constexpr int kRowWarps = kRowThreads / 32;
constexpr int kRowMaxN = 40960;   // keys held in shared memory
constexpr int kRowCandCap = 4096; // keys of the threshold bin kept for digits 2-3

struct RowSmem {
  uint32_t hist[kBins1];
  uint32_t cand[kRowCandCap];
  uint32_t warp_tot[kRowWarps];
  uint64_t warp_tot64[kRowWarps];
  uint32_t bcast[4];
  uint32_t ccount;
};
constexpr size_t kRowKeysOff = (sizeof(RowSmem) + 15) / 16 * 16;

__device__ __forceinline__ uint32_t row_block_sum(RowSmem& sm, uint32_t x) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  if (lane == 0) sm.warp_tot[warp] = x;
  __syncthreads();
  uint32_t s = 0;
  for (int i = 0; i < kRowWarps; ++i) s += sm.warp_tot[i];
  __syncthreads();
  return s;
}

__device__ __forceinline__ int row_find_bin(RowSmem& sm, int nbins, uint32_t need, uint32_t* above) {
  const int per = nbins / kRowThreads;  // 4 or 1
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
  if (lane == 0) sm.warp_tot[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    const uint32_t tw = sm.warp_tot[lane];
    uint32_t ti = tw;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_down_sync(0xffffffffu, ti, o);
      if (lane + o < 32) ti += y;
    }
    sm.warp_tot[lane] = ti - tw;
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

__global__ void __launch_bounds__(kRowThreads, 1)
topk_row_kernel(const float* __restrict__ scores, int64_t n, int64_t row_stride, const int32_t* __restrict__ row_valid,
                const int32_t* __restrict__ id_map, int64_t id_map_stride, int k, int32_t* __restrict__ idx) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  RowSmem& sm = *reinterpret_cast<RowSmem*>(smem_raw);
  uint32_t* keys = reinterpret_cast<uint32_t*>(smem_raw + kRowKeysOff);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t t = blockIdx.x;
  const float* row = scores + t * row_stride;
  const int32_t* idrow = id_map ? id_map + t * id_map_stride : nullptr;
  int32_t* out = idx + t * k;
  int64_t nt64 = n;
  if (row_valid) {
    const int64_t rv = row_valid[t];
    nt64 = rv < 0 ? 0 : (rv < n ? rv : n);
  }
  const int nt = static_cast<int>(nt64);

  for (int i = tid; i < kBins1; i += kRowThreads) sm.hist[i] = 0;
  if (tid == 0) sm.ccount = 0;
  __syncthreads();
  // ---------------- load the row once (4 x 16 B in flight per thread), digit 1
  {
    const int nv = nt / 4;
    const float4* r4 = reinterpret_cast<const float4*>(row);
    for (int i0 = tid; i0 < nv; i0 += 4 * kRowThreads) {
      float4 f[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = i0 + u * kRowThreads;
        f[u] = i < nv ? __ldg(r4 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = i0 + u * kRowThreads;
        if (i < nv) {
          const uint32_t kk[4] = {sel_key(f[u].x), sel_key(f[u].y), sel_key(f[u].z), sel_key(f[u].w)};
          *reinterpret_cast<uint4*>(&keys[4 * i]) = make_uint4(kk[0], kk[1], kk[2], kk[3]);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            if (kk[e]) atomicAdd(&sm.hist[kk[e] >> 20], 1u);
        }
      }
    }
    for (int i = 4 * nv + tid; i < nt; i += kRowThreads) {
      const uint32_t kk = sel_key(__ldg(row + i));
      keys[i] = kk;
      if (kk) atomicAdd(&sm.hist[kk >> 20], 1u);
    }
  }
  __syncthreads();
  uint32_t total;
  {
    uint32_t local = 0;
    for (int i = tid; i < kBins1; i += kRowThreads) local += sm.hist[i];
    total = row_block_sum(sm, local);
  }
  uint32_t tau, need_eq;
  if (total <= static_cast<uint32_t>(k)) {
    tau = kNegInfKey;
    need_eq = 0;
  } else {
    uint32_t gt1, gt2, gt3;
    const int b1 = row_find_bin(sm, kBins1, static_cast<uint32_t>(k), &gt1);
    const uint32_t need1 = static_cast<uint32_t>(k) - gt1;
    // ---------------- digit 2 over the keys of bin b1; keep them as candidates
    for (int i = tid; i < kBins2; i += kRowThreads) sm.hist[i] = 0;
    __syncthreads();
    for (int i = tid; i < nt; i += kRowThreads) {
      const uint32_t kk = keys[i];
      if (kk && static_cast<int>(kk >> 20) == b1) {
        atomicAdd(&sm.hist[(kk >> 10) & 0x3ffu], 1u);
        const uint32_t slot = atomicAdd(&sm.ccount, 1u);
        if (slot < kRowCandCap) sm.cand[slot] = kk;
      }
    }
    __syncthreads();
    const int b2 = row_find_bin(sm, kBins2, need1, &gt2);
    const uint32_t need2 = need1 - gt2;
    const uint32_t pre22 = (static_cast<uint32_t>(b1) << 10) | static_cast<uint32_t>(b2);
    // ---------------- digit 3 over the candidates (or the whole row if they overflowed)
    const uint32_t nc = sm.ccount;
    for (int i = tid; i < kBins2; i += kRowThreads) sm.hist[i] = 0;
    __syncthreads();
    if (nc <= static_cast<uint32_t>(kRowCandCap)) {
      for (uint32_t i = tid; i < nc; i += kRowThreads) {
        const uint32_t kk = sm.cand[i];
        if ((kk >> 10) == pre22) atomicAdd(&sm.hist[kk & 0x3ffu], 1u);
      }
    } else {
      for (int i = tid; i < nt; i += kRowThreads) {
        const uint32_t kk = keys[i];
        if (kk && (kk >> 10) == pre22) atomicAdd(&sm.hist[kk & 0x3ffu], 1u);
      }
    }
    __syncthreads();
    const int b3 = row_find_bin(sm, kBins2, need2, &gt3);
    tau = (pre22 << 10) | static_cast<uint32_t>(b3);
    need_eq = need2 - gt3;
  }

  // ---------------- ordered emission: warp w owns a contiguous chunk
  const int chunk = ((nt + kRowWarps - 1) / kRowWarps + 31) / 32 * 32;
  const int c0 = warp * chunk < nt ? warp * chunk : nt;
  const int c1 = c0 + chunk < nt ? c0 + chunk : nt;
  uint32_t a_cnt = 0, e_cnt = 0;
  for (int i = c0 + lane; i < c1; i += 32) {
    const uint32_t kk = keys[i];
    a_cnt += kk > tau ? 1u : 0u;
    e_cnt += (kk && kk == tau) ? 1u : 0u;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    a_cnt += __shfl_xor_sync(0xffffffffu, a_cnt, o);
    e_cnt += __shfl_xor_sync(0xffffffffu, e_cnt, o);
  }
  if (lane == 0) sm.warp_tot64[warp] = static_cast<uint64_t>(a_cnt) | (static_cast<uint64_t>(e_cnt) << 32);
  __syncthreads();
  if (warp == 0) {
    const uint64_t tw = sm.warp_tot64[lane];
    uint64_t ti = tw;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint64_t y = __shfl_up_sync(0xffffffffu, ti, o);
      if (lane >= o) ti += y;
    }
    sm.warp_tot64[lane] = ti - tw;
    if (lane == 31) {
      sm.bcast[2] = static_cast<uint32_t>(ti & 0xffffffffull);
      sm.bcast[3] = static_cast<uint32_t>(ti >> 32);
    }
  }
  __syncthreads();
  uint32_t a_pos = static_cast<uint32_t>(sm.warp_tot64[warp] & 0xffffffffull);
  uint32_t e_pos = static_cast<uint32_t>(sm.warp_tot64[warp] >> 32);
  const uint32_t lt = (1u << lane) - 1u;
  for (int i0 = c0; i0 < c1; i0 += 32) {
    const int i = i0 + lane;
    const uint32_t kk = i < c1 ? keys[i] : 0u;
    const bool is_a = kk > tau;
    const bool is_e = kk && kk == tau;
    const uint32_t ba = __ballot_sync(0xffffffffu, is_a);
    const uint32_t be = __ballot_sync(0xffffffffu, is_e);
    const uint32_t my_a = a_pos + __popc(ba & lt);
    const uint32_t my_e = e_pos + __popc(be & lt);
    if (is_a) out[my_a + (my_e < need_eq ? my_e : need_eq)] = idrow ? idrow[i] : i;
    else if (is_e && my_e < need_eq) out[my_a + my_e] = idrow ? idrow[i] : i;
    a_pos += __popc(ba);
    e_pos += __popc(be);
  }
  const uint32_t a_all = sm.bcast[2], e_all = sm.bcast[3];
  const uint32_t chosen = a_all + (e_all < need_eq ? e_all : need_eq);
  for (uint32_t i = chosen + tid; i < static_cast<uint32_t>(k); i += kRowThreads) out[i] = -1;
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
    const size_t smem = kRowKeysOff + static_cast<size_t>((n + 3) / 4 * 4) * 4;
    cudaError_t e = ensure_dynamic_smem(reinterpret_cast<const void*>(topk_row_kernel),
                                        static_cast<int>(kRowKeysOff + static_cast<size_t>(kRowMaxN) * 4));
    if (e != cudaSuccess) return e;
    topk_row_kernel<<<T, kRowThreads, smem, stream>>>(scores, n, row_stride, row_valid, id_map, id_map_stride, k, idx);
    return cudaGetLastError();
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

  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(CL, T, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CL;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (in_smem)
    e = cudaLaunchKernelEx(&cfg, topk_cluster_kernel<true>, scores, n, row_stride, row_valid, id_map, id_map_stride, k,
                           idx, slice);
  else
    e = cudaLaunchKernelEx(&cfg, topk_cluster_kernel<false>, scores, n, row_stride, row_valid, id_map, id_map_stride,
                           k, idx, slice);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace misa
