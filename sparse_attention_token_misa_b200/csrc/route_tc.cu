// Head router on the 5th-generation tensor cores.
//
// The block statistics may be windows of B keys every S keys (S < B:
// overlapping windows, HISA explainer (zhichai.net), section 七, 潜在改进);
// window j = [j*S, min(j*S + B, L)) and the visibility rule below hold for any
// S <= B.
//
// "MISA: Mixture of Indexer Sparse Attention for Long-Context LLM Inference"
// (gist.science), Methodology: per-head affinities against block-aggregated
// keys are aggregated into an importance per head for the current query (block)
// and the top-h heads are kept.
//
//   importance[g][h] = sum over the queries t of decision g, and over the blocks
//                      j visible to g, of w[t][h] * ReLU(q[t][h] . mean_j)
//
// The contraction q . mean_j is an MMA: M = 128 (query, head) rows of one
// sequence (qpm queries x H heads, zero rows past them), N = 64 blocks per
// tile, K = 128.  The fp32 block means of a tile arrive by one TMA copy; the
// producers split them into bf16 hi = bf16(m) and lo = bf16(m - hi) (together
// about 16 significant bits) and D = q . hi + q . lo accumulates in fp32 in
// TMEM.  When the caller already holds the split (written with the block
// means) the two bf16 tiles arrive by TMA in the MMA's swizzled layout and no
// conversion runs.  The epilogue thread of row (t, h) sums ReLU(D) over the tile's
// visible blocks and multiplies by w[t][h] (no cross-thread reduction); the
// rows of one head are added in shared memory.  Two ways to combine the work
// items (row group, block tile) of one decision:
//  * a cluster of D <= 8 CTAs per decision (small batches: one wave of
//    clusters): each CTA adds its items' contributions in registers, then CTA
//    0 of the cluster sums the D per-CTA importances in rank order through
//    distributed shared memory and selects;
//  * persistent CTAs over all items (large batches): each epilogue thread adds
//    its row's contributions over a run (the CTA's consecutive items of one
//    decision) in a register; at the end of the run the rows of each head are
//    added once and the run's H partial importances stored; the run's item
//    count goes to the decision's counter (one atomic per run); the CTA that
//    completes the count sums the decision's run partials in CTA order.
// Both orders are fixed, so the result is deterministic.  The top-h are taken
// by rank (value desc, ties to the lower head id), ids ascending.
//
// Roles (416 threads): warps 0-3 epilogue (TMEM lane quarter = warp), warp 4
// TMEM allocation + MMA issue, warp 5 lane 0 TMA of the query rows (once per
// row group) and of the mean tiles, warps 6-12 the hi/lo conversion (idle
// when the split comes from memory).
// Waits are bounded and share a CTA-wide abort flag.
#include <cooperative_groups.h>

#include "launch.h"
#include "misa_device.cuh"

namespace misa {

namespace cg = cooperative_groups;

namespace {

constexpr int kRM = 128;                       // MMA M: (query, head) rows
constexpr int kRN = 64;                        // MMA N: blocks per tile
constexpr int kRStages = 2;
constexpr int kREpiThreads = 128;
constexpr int kRConvThreads = 224;             // warps 6-12
constexpr int kRMmaWarp = 4;
constexpr int kRTmaWarp = 5;
constexpr int kRThreads = 416;
constexpr int kRMaxCluster = 8;
constexpr int kRATileBytes = kRM * kD * 2;     // 32 KB of query rows (bf16)
constexpr int kRFTileBytes = kRN * kD * 4;     // 32 KB of fp32 means
constexpr int kRBTileBytes = kRN * kD * 2;     // 16 KB per hi or lo tile
constexpr int kRStageBytes = kRFTileBytes + 2 * kRBTileBytes;
constexpr int kRTmemCols = 2 * kRN;            // two accumulators
constexpr uint32_t kRIdesc = idesc_bf16_f32(kRM, kRN);
constexpr int kROffA = 0;
constexpr int kROffS = kRATileBytes;
constexpr int kROffBar = kROffS + kRStages * kRStageBytes;
constexpr int kRNumBars = 3 * kRStages + 2 + 2 + 3;
constexpr int kROffTmem = kROffBar + kRNumBars * 8;
constexpr int kROffRed = (kROffTmem + 4 + 15) / 16 * 16;       // [128] row contributions
constexpr int kROffImp = kROffRed + kRM * 4;                     // [MISA_MAX_HEADS] decision importances
constexpr int kROffImp2 = kROffImp + MISA_MAX_HEADS * 4;         // [MISA_MAX_HEADS] cluster sums
constexpr int kROffFlag = kROffImp2 + MISA_MAX_HEADS * 4;        // flag, abort, 4 warp counts
constexpr int kTPitch = kRM + 1;                                  // HISA: [kRN][kTPitch] row contributions
constexpr int kROffT = (kROffFlag + 32 + 15) / 16 * 16;
constexpr int kRSmemBytes = kROffT + kRN * kTPitch * 4 + 1024;

struct RouteParams {
  const uint16_t* q;
  const float* w;
  int64_t means_seq_rows;    // rows of 128 means between sequences in the TMA map
  bool presplit;             // mean tiles given as bf16 hi / lo (else fp32, split here)
  int nseq;
  const int32_t* seq_of;
  const int32_t* prefix_len;
  int T, H;
  int64_t L;
  int B, S, M, q_block, h;  // window length, stride (S = B: plain blocks), windows per sequence
  int qpm;        // queries per row group (share one sequence and one decision)
  int n_pg;       // row groups
  int n_bt;       // block tiles
  int64_t n_items;
  float* partial;            // [n_items][H] partial importances per work item
  unsigned* counters;        // [G] items finished per decision (zero on entry)
  int32_t* heads;            // [G][h]
  float* importance;         // [G][H] or NULL
  float* bscore;             // HISA block scores [T][bs_stride]
  int64_t bs_stride;
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

// number of windows visible to decision g (whole windows inside the prefix of
// its first query): window j = [j*S, min(j*S + B, L)) is visible iff
// min(j*S + B, L) <= prefix, so for a prefix shorter than L the visible
// windows are j <= (prefix - B) / S (S = B: prefix / B whole blocks)
__device__ __forceinline__ int visible_blocks(const RouteParams& p, int g) {
  const int64_t pl = p.prefix_len[static_cast<int64_t>(g) * p.q_block];
  if (pl >= p.L) return p.M;
  if (pl < p.B) return 0;
  const int64_t n = (pl - p.B) / p.S + 1;
  return static_cast<int>(n < p.M ? n : p.M);
}

// Top-h of imp[0, H) (value desc, ties to the lower id; NaN ranks as -inf),
// ids ascending into heads[g].  The 128 epilogue threads call it; thread i
// ranks head i by counting.  wcnt: 4 words of shared memory.
__device__ void select_top_h(const float* imp, int H, int h, int g, int32_t* heads, float* importance,
                             uint32_t* wcnt) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float kNegInf = -__int_as_float(0x7f800000);
  bool sel = false;
  if (tid < H) {
    float x = imp[tid];
    if (importance) importance[static_cast<int64_t>(g) * H + tid] = x;
    x = x == x ? x : kNegInf;
    int rk = 0;
    for (int j = 0; j < H; ++j) {
      float y = imp[j];
      y = y == y ? y : kNegInf;
      rk += (y > x || (y == x && j < tid)) ? 1 : 0;
    }
    sel = rk < h;
  }
  const unsigned m = __ballot_sync(0xffffffffu, sel);
  if (lane == 0) wcnt[warp] = static_cast<uint32_t>(__popc(m));
  named_bar_sync(2, kREpiThreads);
  int before = 0;
  for (int w2 = 0; w2 < warp; ++w2) before += static_cast<int>(wcnt[w2]);
  const int pos = before + __popc(m & ((1u << lane) - 1u));
  if (sel && pos < h) heads[static_cast<int64_t>(g) * h + pos] = tid;
}

// kHisa: the same MMAs give the HISA block scores instead: per (query, block)
// the sum over heads of w * ReLU(q . mean), written out per block tile (no
// reduction across work items).
template <bool kCluster, bool kHisa>
__global__ void __launch_bounds__(kRThreads, 1)
route_tc_kernel(const __grid_constant__ CUtensorMap means_map, const __grid_constant__ CUtensorMap hi_map,
                const __grid_constant__ CUtensorMap lo_map, const __grid_constant__ CUtensorMap q_map,
                const RouteParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem + kROffA;
  uint8_t* sS = smem + kROffS;  // stage s: [fp32 means | hi | lo]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kROffBar);
  uint64_t* ffull = bars;                    // [S] mean tile(s) landed (TMA)
  uint64_t* bfull = bars + kRStages;         // [S] hi/lo tile written
  uint64_t* empty = bars + 2 * kRStages;     // [S] MMAs of the stage done
  uint64_t* tfull = bars + 3 * kRStages;     // [2]
  uint64_t* tempty = bars + 3 * kRStages + 2;
  uint64_t* afull = bars + 3 * kRStages + 4;
  uint64_t* aempty = bars + 3 * kRStages + 5;
  uint64_t* done = bars + 3 * kRStages + 6;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kROffTmem);
  float* red = reinterpret_cast<float*>(smem + kROffRed);
  float* imp = reinterpret_cast<float*>(smem + kROffImp);
  float* imp2 = reinterpret_cast<float*>(smem + kROffImp2);
  unsigned* flag = reinterpret_cast<unsigned*>(smem + kROffFlag);
  volatile uint32_t* abort = reinterpret_cast<volatile uint32_t*>(smem + kROffFlag + 4);
  uint32_t* wcnt = reinterpret_cast<uint32_t*>(smem + kROffFlag + 16);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int s = 0; s < kRStages; ++s) {
      mbar_init(&ffull[s], 1);
      mbar_init(&bfull[s], kRConvThreads);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], kREpiThreads);
    }
    mbar_init(afull, 1);
    mbar_init(aempty, 1);
    mbar_init(done, 1);
    *abort = 0u;
    fence_mbar_init();
  }
  if (warp == kRMmaWarp) {
    tmem_alloc(tmem_slot, kRTmemCols);
    tmem_relinquish();
  }
  if (tid == kRTmaWarp * 32) {
    if (p.presplit) {
      tma_prefetch_desc(&hi_map);
      tma_prefetch_desc(&lo_map);
    } else {
      tma_prefetch_desc(&means_map);
    }
    tma_prefetch_desc(&q_map);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait_inputs();
  pdl_allow_next();

  const int nbt = p.n_bt;
  const int pgs_per_dec = p.q_block / p.qpm;
  int64_t i0, i1;
  int crank = 0, csize = 1, cdec = 0;
  if constexpr (kCluster) {
    // the items of decision cdec, split over the D CTAs of its cluster
    cg::cluster_group cl = cg::this_cluster();
    csize = static_cast<int>(cl.num_blocks());
    crank = static_cast<int>(cl.block_rank());
    cdec = static_cast<int>(blockIdx.x) / csize;
    const int first_pg = cdec * pgs_per_dec;
    const int end_pg = first_pg + pgs_per_dec < p.n_pg ? first_pg + pgs_per_dec : p.n_pg;
    const int64_t first_item = static_cast<int64_t>(first_pg) * nbt;
    const int64_t cnt = (end_pg > first_pg ? static_cast<int64_t>(end_pg - first_pg) * nbt : 0);
    i0 = first_item + cnt * crank / csize;
    i1 = first_item + cnt * (crank + 1) / csize;
  } else {
    i0 = p.n_items * blockIdx.x / gridDim.x;
    i1 = p.n_items * (blockIdx.x + 1) / gridDim.x;
  }

  if (warp == kRTmaWarp) {
    // ------------------------------------------------------------ query rows and mean tiles by TMA
    if (lane == 0) {
      int64_t it = 0;
      int cur_pg = -1, ng = 0;
      bool a_pending = false;
      for (int64_t item = i0; item < i1; ++item, ++it) {
        const int pg = static_cast<int>(item / nbt);
        const int bt = static_cast<int>(item - static_cast<int64_t>(pg) * nbt);
        if (pg != cur_pg) {
          // the group's 128 query rows (rows past its queries belong to later
          // queries or lie past the tensor: their results are weighted by 0)
          if (ng > 0 && !mbar_wait(aempty, (ng - 1) & 1, p.err, abort)) break;
          mbar_arrive_expect_tx(afull, kRATileBytes);
          const int ya = pg * p.qpm * p.H;
          tma_load_2d(sA, &q_map, afull, 0, ya);
          tma_load_2d(sA + kRATileBytes / 2, &q_map, afull, 64, ya);
          a_pending = true;
          cur_pg = pg;
          ++ng;
        }
        const int s = static_cast<int>(it % kRStages);
        const uint32_t ph = static_cast<uint32_t>((it / kRStages) & 1);
        if (!mbar_wait(&empty[s], ph ^ 1u, p.err, abort)) break;
        const int y = static_cast<int>(group_seq(p, pg) * p.means_seq_rows + static_cast<int64_t>(bt) * kRN);
        if (p.presplit) {
          // hi and lo straight into the MMA operand slots, two 64-column halves each
          uint8_t* hi_t = sS + s * kRStageBytes + kRFTileBytes;
          mbar_arrive_expect_tx(&ffull[s], 2 * kRBTileBytes);
          tma_load_2d(hi_t, &hi_map, &ffull[s], 0, y);
          tma_load_2d(hi_t + kRN * 128, &hi_map, &ffull[s], 64, y);
          tma_load_2d(hi_t + kRBTileBytes, &lo_map, &ffull[s], 0, y);
          tma_load_2d(hi_t + kRBTileBytes + kRN * 128, &lo_map, &ffull[s], 64, y);
        } else {
          mbar_arrive_expect_tx(&ffull[s], kRFTileBytes);
          tma_load_2d(sS + s * kRStageBytes, &means_map, &ffull[s], 0, y);
        }
      }
      // no TMA write may still be in flight when the CTA exits
      const int64_t first = it > kRStages ? it - kRStages : 0;
      for (int64_t k2 = first; k2 < it; ++k2)
        mbar_wait(&ffull[k2 % kRStages], static_cast<uint32_t>((k2 / kRStages) & 1), p.err);
      if (a_pending && ng > 0) mbar_wait(afull, (ng - 1) & 1, p.err);
    }
  } else if (warp > kRTmaWarp) {
    // ------------------------------------------------------------ hi/lo conversion
    const int ct = tid - (kRTmaWarp + 1) * 32;
    int64_t it = 0;
    for (int64_t item = i0; !p.presplit && item < i1; ++item, ++it) {
      const int s = static_cast<int>(it % kRStages);
      const uint32_t ph = static_cast<uint32_t>((it / kRStages) & 1);
      if (!mbar_wait(&ffull[s], ph, p.err, abort)) break;
      const float* ft = reinterpret_cast<const float*>(sS + s * kRStageBytes);
      uint8_t* hi_t = sS + s * kRStageBytes + kRFTileBytes;
      uint8_t* lo_t = hi_t + kRBTileBytes;
      for (int x = ct; x < kRN * 16; x += kRConvThreads) {
        const int r = x >> 4, ch = x & 15;
        const float4 a0 = *reinterpret_cast<const float4*>(ft + r * kD + ch * 8);
        const float4 a1 = *reinterpret_cast<const float4*>(ft + r * kD + ch * 8 + 4);
        const float e[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
        uint32_t hw[4], lw[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const __nv_bfloat16 h0 = __float2bfloat16_rn(e[2 * c]);
          const __nv_bfloat16 h1 = __float2bfloat16_rn(e[2 * c + 1]);
          const __nv_bfloat16 l0 = __float2bfloat16_rn(e[2 * c] - __bfloat162float(h0));
          const __nv_bfloat16 l1 = __float2bfloat16_rn(e[2 * c + 1] - __bfloat162float(h1));
          hw[c] = static_cast<uint32_t>(__bfloat16_as_ushort(h0)) | (static_cast<uint32_t>(__bfloat16_as_ushort(h1)) << 16);
          lw[c] = static_cast<uint32_t>(__bfloat16_as_ushort(l0)) | (static_cast<uint32_t>(__bfloat16_as_ushort(l1)) << 16);
        }
        const uint32_t off = sw128_tile_offset(kRN, r, ch);
        *reinterpret_cast<uint4*>(hi_t + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
        *reinterpret_cast<uint4*>(lo_t + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
      }
      fence_proxy_async_smem();
      mbar_arrive(&bfull[s]);
    }
  } else if (warp == kRMmaWarp) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      int64_t it = 0;
      int cur_pg = -1, ng = 0;
      const uint32_t a_addr = smem_u32(sA);
      uint64_t* bready = p.presplit ? ffull : bfull;  // hi/lo tiles of a stage in place
      for (int64_t item = i0; item < i1; ++item, ++it) {
        const int pg = static_cast<int>(item / nbt);
        if (pg != cur_pg) {
          if (!mbar_wait(afull, ng & 1, p.err, abort)) break;
          cur_pg = pg;
          ++ng;
        }
        const int a = static_cast<int>(it & 1);
        const uint32_t aph = static_cast<uint32_t>((it >> 1) & 1);
        if (!mbar_wait(&tempty[a], aph ^ 1u, p.err, abort)) break;
        const int s = static_cast<int>(it % kRStages);
        const uint32_t ph = static_cast<uint32_t>((it / kRStages) & 1);
        if (!mbar_wait(&bready[s], ph, p.err, abort)) break;
        tc_fence_after();
        const uint32_t hi_addr = smem_u32(sS + s * kRStageBytes + kRFTileBytes);
        const uint32_t lo_addr = hi_addr + kRBTileBytes;
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(a * kRN);
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint32_t aoff = (kk >> 2) * (kRM * 128) + (kk & 3) * 32;
          const uint32_t boff = (kk >> 2) * (kRN * 128) + (kk & 3) * 32;
          const uint64_t adesc = sw128_kmajor_desc(a_addr + aoff);
          umma_bf16(d_tmem, adesc, sw128_kmajor_desc(hi_addr + boff), kRIdesc, kk > 0 ? 1u : 0u);
          umma_bf16(d_tmem, adesc, sw128_kmajor_desc(lo_addr + boff), kRIdesc, 1u);
        }
        umma_commit(&empty[s]);
        const bool group_ends = (item + 1 == i1) || (static_cast<int>((item + 1) / nbt) != pg);
        if (group_ends) umma_commit(aempty);
        umma_commit(&tfull[a]);
      }
      umma_commit(done);
      mbar_wait(done, 0, p.err);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    // After a wait gives up the loop keeps running without work ("skip"), so
    // every epilogue thread still reaches every named barrier.
    const int r = warp * 32 + lane;  // row (ql, hh) of the group
    const uint32_t t_lane = tmem_base + (static_cast<uint32_t>(warp * 32) << 16);
    int64_t it = 0;
    float acc = 0.f;  // cluster mode: this CTA's importance of head tid
    int cur_pg = -1;
    float wrow = 0.f;
    int nvis = 0, g = 0;
    int64_t run_items = 0;  // items of decision g done by this CTA since the last counter update
    int64_t run_first = i0;  // first item of the current run (this CTA's consecutive items of one decision)
    float racc = 0.f;        // this row's contributions over the run, in item order
    bool skip = false;
    for (int64_t item = i0; item < i1; ++item, ++it) {
      const int pg = static_cast<int>(item / nbt);
      const int bt = static_cast<int>(item - static_cast<int64_t>(pg) * nbt);
      if (pg != cur_pg) {
        cur_pg = pg;
        g = (pg * p.qpm) / p.q_block;
        nvis = visible_blocks(p, g);
        const int ql = r / p.H, hh = r - ql * p.H;
        const int t = pg * p.qpm + ql;
        wrow = (ql < p.qpm && t < p.T) ? p.w[static_cast<int64_t>(t) * p.H + hh] : 0.f;
      }
      const int a = static_cast<int>(it & 1);
      const uint32_t aph = static_cast<uint32_t>((it >> 1) & 1);
      if constexpr (kHisa) {
        // rows (ql, hh) of the tile through shared memory, then each (query
        // ql, block jj) pair adds its query's heads in ascending order
        float* tb = reinterpret_cast<float*>(smem + kROffT);
        if (!skip && mbar_wait(&tfull[a], aph, p.err, abort)) {
          tc_fence_after();
          uint32_t v[kRN];
#pragma unroll
          for (int u = 0; u < kRN / 16; ++u) tmem_ld16(t_lane + static_cast<uint32_t>(a * kRN + 16 * u), v + 16 * u);
          tmem_wait_ld();
          tc_fence_before();
          mbar_arrive(&tempty[a]);
#pragma unroll
          for (int jj = 0; jj < kRN; ++jj) tb[jj * kTPitch + r] = wrow * fmaxf(__uint_as_float(v[jj]), 0.f);
        } else {
          skip = true;
        }
        named_bar_sync(1, kREpiThreads);
        for (int x = tid; !skip && x < p.qpm * kRN; x += kREpiThreads) {
          const int ql = x / kRN, jj = x - ql * kRN;
          const int t = pg * p.qpm + ql;
          const int64_t j = static_cast<int64_t>(bt) * kRN + jj;
          if (t < p.T && j < p.M) {
            float sum = 0.f;
            for (int hh = 0; hh < p.H; ++hh) sum += tb[jj * kTPitch + ql * p.H + hh];
            // wholly visible: the score; cut by the prefix (the query's own
            // block): +inf, always kept; later: -inf
            const int64_t plen = p.prefix_len[t];
            const int64_t start = j * p.S;
            const int64_t end = start + p.B < p.L ? start + p.B : p.L;
            const float inf = __int_as_float(0x7f800000);
            p.bscore[static_cast<int64_t>(t) * p.bs_stride + j] =
                end <= plen ? sum : ((start < plen && plen < end) ? inf : -inf);
          }
        }
        named_bar_sync(1, kREpiThreads);  // tb is reused by the next item
        continue;
      }
      float contrib = 0.f;
      if (!skip && mbar_wait(&tfull[a], aph, p.err, abort)) {
        tc_fence_after();
        int nc = nvis - bt * kRN;  // visible columns of this tile
        nc = nc < 0 ? 0 : (nc > kRN ? kRN : nc);
        uint32_t v[kRN];
#pragma unroll
        for (int u = 0; u < kRN / 16; ++u) tmem_ld16(t_lane + static_cast<uint32_t>(a * kRN + 16 * u), v + 16 * u);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(&tempty[a]);
        float sum = 0.f;
        if (nc == kRN) {
#pragma unroll
          for (int jj = 0; jj < kRN; ++jj) sum += fmaxf(__uint_as_float(v[jj]), 0.f);
        } else {
#pragma unroll
          for (int jj = 0; jj < kRN; ++jj) sum += jj < nc ? fmaxf(__uint_as_float(v[jj]), 0.f) : 0.f;
        }
        contrib = wrow * sum;
      } else {
        skip = true;
      }
      racc += contrib;
      ++run_items;
      // a run ends with this CTA's last item of decision g: only then are the
      // rows of one head added (shared memory) and the run's partial stored
      const bool run_ends = (item + 1 == i1) || (static_cast<int>((((item + 1) / nbt) * p.qpm) / p.q_block) != g);
      if (!run_ends) continue;
      red[r] = racc;
      racc = 0.f;
      named_bar_sync(1, kREpiThreads);
      float hsum = 0.f;
      if (tid < p.H)
        for (int k2 = 0; k2 < p.qpm; ++k2) hsum += red[k2 * p.H + tid];
      if constexpr (kCluster) {
        if (tid < p.H && !skip) acc += hsum;
        run_items = 0;
        run_first = item + 1;
        named_bar_sync(1, kREpiThreads);  // red is reused by the next run
        continue;
      }
      if (tid < p.H && !skip) p.partial[run_first * p.H + tid] = hsum;
      {
        const int first_pg = g * pgs_per_dec;
        const int last_pg = (first_pg + pgs_per_dec < p.n_pg ? first_pg + pgs_per_dec : p.n_pg) - 1;
        const int64_t first_item = static_cast<int64_t>(first_pg) * nbt;
        const int64_t end_item = static_cast<int64_t>(last_pg + 1) * nbt;
        __threadfence();
        named_bar_sync(1, kREpiThreads);
        if (tid == 0) {
          const unsigned expected = static_cast<unsigned>(end_item - first_item);
          flag[0] = (!*abort && atomicAdd(&p.counters[g], static_cast<unsigned>(run_items)) +
                                        static_cast<unsigned>(run_items) == expected)
                        ? 1u
                        : 0u;
        }
        named_bar_sync(1, kREpiThreads);
        if (flag[0]) {
          __threadfence();
          if (tid < p.H) {
            // the decision's runs in CTA order: one starts at its first item,
            // the others where the item range of a CTA begins inside it (the
            // grid never exceeds the item count, so those starts are distinct)
            float sum = __ldcg(&p.partial[first_item * p.H + tid]);
            for (int c2 = 1; c2 < static_cast<int>(gridDim.x); ++c2) {
              const int64_t st = p.n_items * c2 / gridDim.x;
              if (st > first_item && st < end_item) sum += __ldcg(&p.partial[st * p.H + tid]);
            }
            imp[tid] = sum;
          }
          named_bar_sync(1, kREpiThreads);
          select_top_h(imp, p.H, p.h, g, p.heads, p.importance, wcnt);
          if (tid == 0) p.counters[g] = 0u;  // ready for the next call
        }
      }
      run_items = 0;
      run_first = item + 1;
      named_bar_sync(1, kREpiThreads);  // red / imp / flag are reused by the next run
    }
    if constexpr (kCluster) {
      if (tid < p.H) imp[tid] = acc;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kRMmaWarp) tmem_dealloc(tmem_base, kRTmemCols);
  if constexpr (kCluster) {
    cg::cluster_group cl = cg::this_cluster();
    cl.sync();  // every CTA's importances are complete
    if (crank == 0 && warp < kREpiThreads / 32) {
      if (tid < p.H) {
        // all reads issued first, then added in rank order
        float part[kRMaxCluster];
#pragma unroll
        for (int c = 0; c < kRMaxCluster; ++c) part[c] = c < csize ? cl.map_shared_rank(imp, c)[tid] : 0.f;
        float sum = 0.f;
#pragma unroll
        for (int c = 0; c < kRMaxCluster; ++c)
          if (c < csize) sum += part[c];
        imp2[tid] = sum;
      }
      named_bar_sync(1, kREpiThreads);
      if (cdec < p.n_pg / pgs_per_dec + (p.n_pg % pgs_per_dec ? 1 : 0))
        select_top_h(imp2, p.H, p.h, cdec, p.heads, p.importance, wcnt);
    }
    cl.sync();  // CTA 0 has read every CTA's importances
  }
}

}  // namespace

int route_tc_queries_per_group(int H, int q_block, bool shared_sequence) {
  if (!shared_sequence) return 1;
  int qpm = 1;
  while (qpm * 2 * H <= kRM && q_block % (qpm * 2) == 0) qpm *= 2;
  return qpm;
}

namespace {

// Tensor maps of the block means: fp32 rows of 128 (one TMA box per tile),
// or, when the split is given, the bf16 hi and lo rows in 128-byte swizzled
// halves (the MMA's B layout).  The maps a launch does not use stay zero.
bool encode_mean_maps(const float* means, const uint16_t* hi, const uint16_t* lo, uint64_t rows, CUtensorMap* fmap,
                      CUtensorMap* hmap, CUtensorMap* lmap) {
  *fmap = CUtensorMap{};
  *hmap = CUtensorMap{};
  *lmap = CUtensorMap{};
  if (hi && lo)
    return encode_2d_map(hmap, true, hi, kD, rows, kD * 2, 64, kRN, true) &&
           encode_2d_map(lmap, true, lo, kD, rows, kD * 2, 64, kRN, true);
  return encode_2d_map(fmap, false, means, kD, rows, kD * 4, kD, kRN, false);
}

}  // namespace

cudaError_t launch_route_heads_tc(const uint16_t* q, const float* w, const float* means, const uint16_t* means_hi,
                                  const uint16_t* means_lo, int64_t means_seq_stride,
                                  int nseq, const int32_t* seq_of, const int32_t* prefix_len, int T, int H, int64_t L,
                                  int B, int S, int q_block, int h, int qpm, int32_t* heads, float* importance,
                                  float* partial, unsigned* counters, bool clear_counters, uint32_t* err,
                                  cudaStream_t stream) {
  RouteParams p = {};
  p.q = q;
  p.w = w;
  p.means_seq_rows = means_seq_stride / kD;
  p.nseq = nseq;
  p.seq_of = seq_of;
  p.prefix_len = prefix_len;
  p.T = T;
  p.H = H;
  p.L = L;
  p.B = B;
  p.S = S;
  p.M = static_cast<int>(num_windows(L, B, S));
  p.q_block = q_block;
  p.h = h;
  p.qpm = qpm;
  p.n_pg = (T + qpm - 1) / qpm;
  p.n_bt = (p.M + kRN - 1) / kRN;
  p.n_items = static_cast<int64_t>(p.n_pg) * p.n_bt;
  p.partial = partial;
  p.counters = counters;
  p.heads = heads;
  p.importance = importance;
  p.err = err;
  p.presplit = means_hi && means_lo;
  // means as rows of 128: sequence b's block j is row b * means_seq_rows + j
  CUtensorMap map, hmap, lmap;
  const uint64_t rows = static_cast<uint64_t>(nseq - 1) * static_cast<uint64_t>(p.means_seq_rows) + p.M;
  if (!encode_mean_maps(means, means_hi, means_lo, rows, &map, &hmap, &lmap)) return cudaErrorInvalidValue;
  // query rows, bf16, 128-byte swizzled K-major like the keys
  CUtensorMap qmap;
  if (!encode_2d_map(&qmap, true, q, kD, static_cast<uint64_t>(T) * H, kD * 2, 64, kRM, true))
    return cudaErrorInvalidValue;
  const int sms = device_sm_count();
  if (sms <= 0) return cudaErrorInvalidDevice;
  // cluster mode when one wave of clusters covers the batch: D CTAs per
  // decision, each with at most 8 items
  const int G = (T + q_block - 1) / q_block;
  const int64_t items_per_dec = static_cast<int64_t>(q_block / qpm) * p.n_bt;
  const int D = static_cast<int>(items_per_dec < kRMaxCluster ? items_per_dec : kRMaxCluster);
  const bool cluster = items_per_dec <= 8 * kRMaxCluster && static_cast<int64_t>(G) * D <= sms;
  cudaError_t e = cudaSuccess;
  if (cluster) {
    e = ensure_dynamic_smem(reinterpret_cast<const void*>(route_tc_kernel<true, false>), kRSmemBytes);
    if (e != cudaSuccess) return e;
    return launch_pdl(route_tc_kernel<true, false>, dim3(static_cast<unsigned>(G * D)), dim3(kRThreads), kRSmemBytes, stream,
                      D, map, hmap, lmap, qmap, p);
  }
  if (clear_counters) {
    e = cudaMemsetAsync(counters, 0, static_cast<size_t>(G) * sizeof(unsigned), stream);
    if (e != cudaSuccess) return e;
  }
  e = ensure_dynamic_smem(reinterpret_cast<const void*>(route_tc_kernel<false, false>), kRSmemBytes);
  if (e != cudaSuccess) return e;
  const int64_t grid = p.n_items < sms ? p.n_items : sms;
  return launch_pdl(route_tc_kernel<false, false>, dim3(static_cast<unsigned>(grid)), dim3(kRThreads), kRSmemBytes, stream, 0,
                    map, hmap, lmap, qmap, p);
}

cudaError_t launch_hisa_block_scores_tc(const uint16_t* q, const float* w, const float* means,
                                        const uint16_t* means_hi, const uint16_t* means_lo, int64_t means_seq_stride, int nseq, const int32_t* seq_of,
                                        const int32_t* prefix_len, int T, int H, int64_t L, int B, int S,
                                        float* bscore, int64_t bs_stride, uint32_t* err, cudaStream_t stream) {
  if (H > kRM) return cudaErrorInvalidValue;
  const bool shared = nseq == 1 || means_seq_stride == 0;
  int qpm = 1;
  while (shared && qpm * 2 * H <= kRM) qpm *= 2;
  RouteParams p = {};
  p.q = q;
  p.w = w;
  p.means_seq_rows = means_seq_stride / kD;
  p.nseq = nseq;
  p.seq_of = seq_of;
  p.prefix_len = prefix_len;
  p.T = T;
  p.H = H;
  p.L = L;
  p.B = B;
  p.S = S;
  p.M = static_cast<int>(num_windows(L, B, S));
  p.q_block = qpm;  // (no routing decisions in this mode)
  p.h = 1;
  p.qpm = qpm;
  p.n_pg = (T + qpm - 1) / qpm;
  p.n_bt = (p.M + kRN - 1) / kRN;
  p.n_items = static_cast<int64_t>(p.n_pg) * p.n_bt;
  p.bscore = bscore;
  p.bs_stride = bs_stride;
  p.err = err;
  p.presplit = means_hi && means_lo;
  CUtensorMap map, hmap, lmap;
  const uint64_t rows = static_cast<uint64_t>(nseq - 1) * static_cast<uint64_t>(p.means_seq_rows) + p.M;
  if (!encode_mean_maps(means, means_hi, means_lo, rows, &map, &hmap, &lmap)) return cudaErrorInvalidValue;
  CUtensorMap qmap;
  if (!encode_2d_map(&qmap, true, q, kD, static_cast<uint64_t>(T) * H, kD * 2, 64, kRM, true))
    return cudaErrorInvalidValue;
  cudaError_t e = ensure_dynamic_smem(reinterpret_cast<const void*>(route_tc_kernel<false, true>), kRSmemBytes);
  if (e != cudaSuccess) return e;
  const int sms = device_sm_count();
  if (sms <= 0) return cudaErrorInvalidDevice;
  const int64_t grid = p.n_items < sms ? p.n_items : sms;
  return launch_pdl(route_tc_kernel<false, true>, dim3(static_cast<unsigned>(grid)), dim3(kRThreads), kRSmemBytes,
                    stream, 0, map, hmap, lmap, qmap, p);
}

}  // namespace misa
