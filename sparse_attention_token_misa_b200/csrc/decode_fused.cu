// Router and routed token scoring of a MISA decode step in one kernel.
//
// "MISA: Mixture of Indexer Sparse Attention for Long-Context LLM Inference"
// (gist.science), Methodology: a router scores the heads against mean-pooled
// key blocks and keeps h of the H indexer heads for the current query; only
// those heads score every prefix token; the top-k tokens are kept.  The
// library's definitions (misa.h): A[t,h,j] = w[t,h] * ReLU(q[t,h] . mean_j),
// importance = sum over visible blocks, top-h by rank (ties to the lower head),
// S[t,s] = sum over the routed heads of w * ReLU(q . k_s).  The top-k of the
// score rows is the top-k kernel's, launched right behind this one (topk.cu).
//
// Why one kernel: at decode the step is one pass over the keys (HBM-bound),
// and the router is a short chain of dependent steps that leaves HBM idle when
// it runs as a kernel of its own.  Here every CTA starts its key stream as
// soon as its first router tiles are on their way, and routes the queries it
// works on from a buffer of its own while the key tiles land.
//
// Work: one persistent CTA per SM over the items (query g, key tile j) in
// contiguous ranges, exactly as the scoring kernel splits them.  Per query the
// CTA touches:
//  * router: the bf16 hi / lo block means of the query's cache arrive by TMA
//    in a two-slot router buffer (128 blocks x 128 dims per tile: the MMA's A
//    operand, blocks are the M = 128 rows), the query's H rows are the B
//    operand (N = NR columns); D = q . hi + q . lo accumulates in TMEM (two
//    accumulators).  Four router warps read them: each thread holds one
//    block's affinities, applies ReLU and the visibility mask; a butterfly over
//    the lanes leaves each lane with NR / 32 heads' sums, the warps add in
//    fixed order in shared memory, the block tiles add up in order, the head
//    weight multiplies once, and the top-h are ranked.  Every CTA that works on
//    a query computes the same heads (same data, same instruction order).  The
//    next query's router MMAs are issued between the current query's scoring
//    MMAs as soon as their operands land, so the key stream does not wait.
//  * scoring: the routed rows (h <= 16, zero padded to N = 16) are copied from
//    the query rows already in shared memory into the B operand; the key tiles
//    stream through a four-stage ring; the scoring epilogue is the scoring
//    kernel's (ReLU, head weights, heads summed in ascending order), so the
//    scores equal misa_index_score's bit for bit given the same heads.  The
//    score rows stay in L2 for the top-k kernel.
//
// Roles (352 threads): warps 0-3 scoring epilogue (TMEM lane quarter = warp),
// warps 4-7 router epilogue (lane quarter = warp - 4), warp 8 TMEM allocation
// + single-thread MMA issue, warp 9 one thread for the key tiles, warp 10 one
// thread for the query rows and router tiles.  Every wait is bounded; a wait
// that gives up records MISA_DEVERR_TIMEOUT, raises a CTA-wide abort flag and
// the roles stop; TMEM is freed before exit.
#include <algorithm>
#include <cstring>

#include "launch.h"
#include "misa_device.cuh"

namespace misa {

namespace {

constexpr int kFTileM = 128;                    // keys (or blocks) per tile
constexpr int kFTileBytes = kFTileM * kD * 2;   // 32 KB
constexpr int kFStages = 4;                     // key ring
constexpr int kFPrefetch = kFStages + 2;        // key tiles asked into L2 this far ahead
constexpr int kFRSlots = 2;                     // router buffer (hi / lo tiles)
constexpr int kFHP = 16;                        // routed columns (h <= 16, zero padded)
constexpr int kFThreads = 352;
constexpr int kFEpiThreads = 128;               // scoring epilogue (warps 0-3)
constexpr int kFRouteWarp0 = 4;                 // router epilogue (warps 4-7)
constexpr int kFMmaWarp = 8;
constexpr int kFKeyWarp = 9;
constexpr int kFRouterTmaWarp = 10;
constexpr int kFMaxL = 65536;                   // longest row
constexpr int kFMaxNR = 64;                     // router columns (H <= 64)
constexpr int kFTmemCols = 256;                 // 2 router accumulators (<= 64 each) + 2 x 16 scoring

// shared memory map (offsets from a 1024-byte aligned base)
constexpr int kFOffRing = 0;                                      // [4] key tiles
constexpr int kFOffRBuf = kFOffRing + kFStages * kFTileBytes;     // [2] router tiles
constexpr int kFOffQall = kFOffRBuf + kFRSlots * kFTileBytes;     // [NR rows x 128] router B operand
constexpr int kFOffSQ = kFOffQall + kFMaxNR * kD * 2;             // 2 x [16 rows x 128] scoring B operand
constexpr int kFSQBytes = kFHP * kD * 2;                          // 4 KB
constexpr int kFOffRed = kFOffSQ + 2 * kFSQBytes;                 // [4][64] f32 router warp partial sums
constexpr int kFOffImp = kFOffRed + 4 * kFMaxNR * 4;              // [64] f32 head sums
constexpr int kFOffHeads = kFOffImp + kFMaxNR * 4;                // [16] i32 routed heads (router epilogue)
constexpr int kFOffW = kFOffHeads + kFHP * 4;                     // [2][16] f32 routed weights
constexpr int kFOffMisc = kFOffW + 2 * kFHP * 4;                  // [64] u32 scratch words
constexpr int kFOffBar = kFOffMisc + 64 * 4;
// full[4] empty[4] rbfull[2] rbempty[2] qa_full qa_empty, then pairs rfull
// rempty tfull tempty qfull qempty wempty, then done
constexpr int kFNumBars = 2 * kFStages + 2 * kFRSlots + 2 + 2 * 7 + 1;
constexpr int kFOffTmem = kFOffBar + kFNumBars * 8;
constexpr int kFSmemBytes = kFOffTmem + 16 + 1024;                // + alignment slack
static_assert(kFSmemBytes <= 232448, "shared memory per CTA");

struct FusedParams {
  const uint16_t* q;
  const float* w;
  const int32_t* seq_of;
  const int32_t* prefix_len;
  int T, H, h;
  int64_t L;
  int B, M, n_rt;           // block size, blocks per sequence, router tiles (128 blocks) per query
  int64_t key_seq_rows;     // key rows between sequences in the key map
  int64_t mean_seq_rows;    // mean rows between sequences in the hi / lo maps
  int64_t nkeyseq, nmeanseq;
  int tpg;                  // key tiles per query
  int64_t n_items;
  int32_t* heads;           // [T][h] out
  float* importance;        // [T][H] out or NULL
  float* scores;            // [T][row_stride] out
  int64_t row_stride;
  uint32_t* err;
};

__device__ __forceinline__ int64_t f_item_begin(int64_t n_items, int c, int G) { return n_items * c / G; }

__device__ __forceinline__ int f_seq_checked(const FusedParams& p, int g, int64_t nseq) {
  int64_t s = p.seq_of[g];
  if (s < 0 || s >= nseq) {
    record_error(p.err, MISA_DEVERR_BAD_SEQ);
    s = 0;
  }
  return static_cast<int>(s);
}

__device__ __forceinline__ int f_valid_len(const FusedParams& p, int g) {
  int64_t pl = p.prefix_len[g];
  if (pl > p.L) pl = p.L;
  if (pl < 0) pl = 0;
  return static_cast<int>(pl);
}

// whole blocks inside the prefix (all M at decode)
__device__ __forceinline__ int f_visible_blocks(const FusedParams& p, int g) {
  const int64_t pl = p.prefix_len[g];
  if (pl >= p.L) return p.M;
  if (pl <= 0) return 0;
  return static_cast<int>(pl / p.B);
}

// Sum over the lanes of a warp of NR per-lane values (one per head), leaving
// lane l with heads [base, base + NR / 32) (NR >= 32) or head l >> 1 (NR = 16,
// held by both lanes of a pair).  Butterfly: each step keeps one half of the
// values and adds the partner's copy of it, so no value crosses more than once.
template <int NR>
__device__ __forceinline__ void f_lane_reduce(float (&v)[NR], int lane) {
#pragma unroll
  for (int step = 0; step < 5; ++step) {
    const int o = 16 >> step;
    const int width = NR >> step;  // values still held
    if (width > 1) {
      const bool upper = (lane >> (4 - step)) & 1;
#pragma unroll
      for (int i = 0; i < (NR >> (step + 1)); ++i) {
        const float a = v[i], b = v[i + (NR >> (step + 1))];
        const float send = upper ? a : b;
        const float keep = upper ? b : a;
        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
      }
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], o);
    }
  }
}

// First head index lane `lane` holds after f_lane_reduce, and how many.
template <int NR>
__device__ __forceinline__ int f_lane_head0(int lane) {
  return NR >= 32 ? lane * (NR / 32) : (lane >> 1);
}
template <int NR>
constexpr int f_lane_heads() {
  return NR >= 32 ? NR / 32 : 1;
}

template <int NR>
__global__ void __launch_bounds__(kFThreads, 1)
decode_fused_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap hmap,
                    const __grid_constant__ CUtensorMap lmap, const __grid_constant__ CUtensorMap qmap,
                    const FusedParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* ring = smem + kFOffRing;
  uint8_t* rbuf = smem + kFOffRBuf;
  uint8_t* qall = smem + kFOffQall;
  uint8_t* sq = smem + kFOffSQ;
  float* red = reinterpret_cast<float*>(smem + kFOffRed);
  float* imp = reinterpret_cast<float*>(smem + kFOffImp);
  int32_t* heads_r = reinterpret_cast<int32_t*>(smem + kFOffHeads);
  float* w_s = reinterpret_cast<float*>(smem + kFOffW);
  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + kFOffMisc);   // [0,8) router, [63] key-stream start flag
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kFOffBar);
  uint64_t* full = bars;                        // [4] key tile landed
  uint64_t* empty = full + kFStages;            // [4] MMAs reading the key tile done
  uint64_t* rbfull = empty + kFStages;          // [2] router tile landed
  uint64_t* rbempty = rbfull + kFRSlots;        // [2] MMAs reading the router tile done
  uint64_t* qa_full = rbempty + kFRSlots;       // query rows of the router landed
  uint64_t* qa_empty = qa_full + 1;             // router MMAs and routed-row copies done with them
  uint64_t* rfull = qa_full + 2;                // [2] router accumulator ready
  uint64_t* rempty = rfull + 2;                 // [2] router accumulator read
  uint64_t* tfull = rempty + 2;                 // [2] scoring accumulator ready
  uint64_t* tempty = tfull + 2;                 // [2] scoring accumulator read
  uint64_t* qfull = tempty + 2;                 // [2] routed rows and weights staged
  uint64_t* qempty = qfull + 2;                 // [2] MMAs of the query using the staged rows done
  uint64_t* wempty = qempty + 2;                // [2] scoring epilogue took the weights
  uint64_t* done = wempty + 2;
  static_assert(2 * kFStages + 2 * kFRSlots + 2 + 2 * 7 + 1 == kFNumBars, "barrier layout");
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kFOffTmem);
  volatile uint32_t* abort = reinterpret_cast<volatile uint32_t*>(smem + kFOffTmem + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  constexpr uint32_t kIdescR = idesc_bf16_f32(kFTileM, NR);
  constexpr uint32_t kIdescS = idesc_bf16_f32(kFTileM, kFHP);

  if (tid == 0) {
    for (int s = 0; s < kFStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int s = 0; s < kFRSlots; ++s) {
      mbar_init(&rbfull[s], 1);
      mbar_init(&rbempty[s], 1);
    }
    mbar_init(qa_full, 1);
    mbar_init(qa_empty, kFEpiThreads);
    for (int a = 0; a < 2; ++a) {
      mbar_init(&rfull[a], 1);
      mbar_init(&rempty[a], kFEpiThreads);
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], kFEpiThreads);
      mbar_init(&qfull[a], kFEpiThreads);
      mbar_init(&qempty[a], 1);
      mbar_init(&wempty[a], kFEpiThreads);
    }
    mbar_init(done, 1);
    *abort = 0u;
    fence_mbar_init();
  }
  if (tid == 0) misc[63] = 0u;   // router producer -> key producer: the first router loads are issued
  if (warp == kFMmaWarp) {
    tmem_alloc(tmem_slot, kFTmemCols);
    tmem_relinquish();
  }
  if (tid == kFKeyWarp * 32) tma_prefetch_desc(&kmap);
  if (tid == kFRouterTmaWarp * 32) {
    tma_prefetch_desc(&hmap);
    tma_prefetch_desc(&lmap);
    tma_prefetch_desc(&qmap);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait_inputs();
  pdl_allow_next();

  const int G = static_cast<int>(gridDim.x);
  const int c = static_cast<int>(blockIdx.x);
  const int64_t i0 = f_item_begin(p.n_items, c, G), i1 = f_item_begin(p.n_items, c + 1, G);
  const int tpg = p.tpg;
  const int g0 = static_cast<int>(i0 / tpg);
  const int ng = i1 > i0 ? static_cast<int>((i1 - 1) / tpg) - g0 + 1 : 0;   // queries this CTA works on
  auto run_begin = [&](int gl) { return std::max<int64_t>(i0, static_cast<int64_t>(g0 + gl) * tpg); };
  auto run_end = [&](int gl) { return std::min<int64_t>(i1, static_cast<int64_t>(g0 + gl + 1) * tpg); };

  if (warp == kFKeyWarp) {
    // ------------------------------------------------------------ key tiles, from the first cycle
    if (lane == 0) {
      const uint64_t kpol = l2_evict_first_policy();   // keys are read once
      // let the router's first loads go ahead of the key stream (they are on
      // the path to the first scoring MMA); bounded like every wait
      {
        volatile uint32_t* go = misc + 63;
        const uint64_t t0 = globaltimer_ns();
        while (*go == 0u && !*abort && globaltimer_ns() - t0 < kWaitLimitNs) {
        }
      }
      const int64_t krows = (p.nkeyseq - 1) * p.key_seq_rows + p.L;   // rows of the key map
      int64_t it = 0;
      bool ok = true;
      for (int gl = 0; gl < ng && ok; ++gl) {
        const int g = g0 + gl;
        const int kseq = f_seq_checked(p, g, p.nkeyseq);
        for (int64_t item = run_begin(gl); item < run_end(gl) && ok; ++item, ++it) {
          const int j = static_cast<int>(item - static_cast<int64_t>(g) * tpg);
          const int s = static_cast<int>(it % kFStages);
          if (!mbar_wait(&empty[s], static_cast<uint32_t>(((it / kFStages) & 1) ^ 1), p.err, abort)) {
            ok = false;
            break;
          }
          uint8_t* dst = ring + s * kFTileBytes;
          mbar_arrive_expect_tx(&full[s], kFTileBytes);
          const int y = static_cast<int>(kseq * p.key_seq_rows + static_cast<int64_t>(j) * kFTileM);
#pragma unroll
          for (int r0 = 0; r0 < kFTileM; r0 += kTmaBoxRows) {
            tma_load_2d_hint(dst + r0 * 128, &kmap, &full[s], 0, y + r0, kpol);
            tma_load_2d_hint(dst + kFTileBytes / 2 + r0 * 128, &kmap, &full[s], 64, y + r0, kpol);
          }
          // the tile two past the ring's reach is asked into L2 now, so that
          // more of the stream is in flight than the ring holds
          if (item + kFPrefetch < run_end(gl) && j + kFPrefetch < tpg) {
            const int yp = y + kFPrefetch * kFTileM;
            for (int r0 = 0; r0 < kFTileM && yp + r0 < krows; r0 += kTmaBoxRows) {
              tma_prefetch_l2_2d(&kmap, 0, yp + r0);
              tma_prefetch_l2_2d(&kmap, 64, yp + r0);
            }
          }
        }
      }
      // no TMA write may still be in flight when the CTA exits
      const int64_t first = it > kFStages ? it - kFStages : 0;
      for (int64_t k2 = first; k2 < it; ++k2)
        mbar_wait(&full[k2 % kFStages], static_cast<uint32_t>((k2 / kFStages) & 1), p.err);
    }
  } else if (warp == kFRouterTmaWarp) {
    // ------------------------------------------------------------ query rows and router tiles
    if (lane == 0) {
      int64_t rb = 0;
      bool ok = true;
      for (int gl = 0; gl < ng && ok; ++gl) {
        const int g = g0 + gl;
        if (gl > 0 && !mbar_wait(qa_empty, (gl - 1) & 1, p.err, abort)) break;
        mbar_arrive_expect_tx(qa_full, static_cast<uint32_t>(p.H) * kD * 2);
        tma_load_2d(qall, &qmap, qa_full, 0, g * p.H);
        tma_load_2d(qall + NR * 128, &qmap, qa_full, 64, g * p.H);
        const int mseq = f_seq_checked(p, g, p.nmeanseq);
        for (int rt = 0; rt < p.n_rt && ok; ++rt) {
          for (int part = 0; part < 2; ++part, ++rb) {
            const int s = static_cast<int>(rb % kFRSlots);
            if (!mbar_wait(&rbempty[s], static_cast<uint32_t>(((rb / kFRSlots) & 1) ^ 1), p.err, abort)) {
              ok = false;
              break;
            }
            uint8_t* dst = rbuf + s * kFTileBytes;
            const CUtensorMap* mp = part == 0 ? &hmap : &lmap;
            mbar_arrive_expect_tx(&rbfull[s], kFTileBytes);
            const int y = static_cast<int>(mseq * p.mean_seq_rows + static_cast<int64_t>(rt) * kFTileM);
#pragma unroll
            for (int r0 = 0; r0 < kFTileM; r0 += kTmaBoxRows) {
              tma_load_2d(dst + r0 * 128, mp, &rbfull[s], 0, y + r0);
              tma_load_2d(dst + kFTileBytes / 2 + r0 * 128, mp, &rbfull[s], 64, y + r0);
            }
          }
          if (gl == 0 && rt == 0 && ok) {
            // the first pair is on its way: the keys may follow; every later
            // router tile of this CTA's queries is asked into L2 now, so that
            // its load, when its slot frees, is an L2 hit
            *reinterpret_cast<volatile uint32_t*>(misc + 63) = 1u;
            const int64_t mrows = (p.nmeanseq - 1) * p.mean_seq_rows + p.M;   // rows of the hi / lo maps
            for (int gl2 = 0; gl2 < ng && gl2 < 4; ++gl2) {
              const int ms2 = f_seq_checked(p, g0 + gl2, p.nmeanseq);
              for (int rt2 = (gl2 == 0 ? 1 : 0); rt2 < p.n_rt; ++rt2) {
                const int y2 = static_cast<int>(ms2 * p.mean_seq_rows + static_cast<int64_t>(rt2) * kFTileM);
                for (int r0 = 0; r0 < kFTileM && y2 + r0 < mrows; r0 += kTmaBoxRows)
                  for (int x0 = 0; x0 < kD; x0 += 64) {
                    tma_prefetch_l2_2d(&hmap, x0, y2 + r0);
                    tma_prefetch_l2_2d(&lmap, x0, y2 + r0);
                  }
              }
            }
          }
        }
      }
      *reinterpret_cast<volatile uint32_t*>(misc + 63) = 1u;
      const int64_t first = rb > kFRSlots ? rb - kFRSlots : 0;
      for (int64_t k2 = first; k2 < rb; ++k2)
        mbar_wait(&rbfull[k2 % kFRSlots], static_cast<uint32_t>((k2 / kFRSlots) & 1), p.err);
      if (ng > 0) mbar_wait(qa_full, (ng - 1) & 1, p.err);
    }
  } else if (warp == kFMmaWarp) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      const uint32_t qall_addr = smem_u32(qall);
      int64_t it = 0, acc = 0;     // key tiles, scoring accumulators
      int64_t rb = 0, rit = 0;     // router tiles, router accumulators
      int r_gl = 0, r_rt = 0;      // next router pair to issue: query, block tile
      bool ok = true;
      // Issue the next router pair (hi and lo of one 128-block tile) of query
      // r_gl; without `block`, only when its operands have landed.
      auto router_pair = [&](bool block) -> bool {
        const int ab = static_cast<int>(rit & 1);
        const int s0 = static_cast<int>(rb % kFRSlots), s1 = static_cast<int>((rb + 1) % kFRSlots);
        const uint32_t ph0 = static_cast<uint32_t>((rb / kFRSlots) & 1);
        const uint32_t ph1 = static_cast<uint32_t>(((rb + 1) / kFRSlots) & 1);
        const uint32_t rph = static_cast<uint32_t>(((rit >> 1) & 1) ^ 1);
        if (!block && !(mbar_try_wait(qa_full, r_gl & 1) && mbar_try_wait(&rempty[ab], rph) &&
                        mbar_try_wait(&rbfull[s0], ph0) && mbar_try_wait(&rbfull[s1], ph1)))
          return false;
        if (!mbar_wait(qa_full, r_gl & 1, p.err, abort) || !mbar_wait(&rempty[ab], rph, p.err, abort)) {
          ok = false;
          return false;
        }
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(ab * NR);
        for (int part = 0; part < 2; ++part, ++rb) {
          const int s = static_cast<int>(rb % kFRSlots);
          if (!mbar_wait(&rbfull[s], static_cast<uint32_t>((rb / kFRSlots) & 1), p.err, abort)) {
            ok = false;
            return false;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(rbuf + s * kFTileBytes);
#pragma unroll
          for (int kk = 0; kk < kD / 16; ++kk) {
            const uint64_t adesc = sw128_kmajor_desc(a_addr + (kk >> 2) * (kFTileM * 128) + (kk & 3) * 32);
            const uint64_t bdesc = sw128_kmajor_desc(qall_addr + (kk >> 2) * (NR * 128) + (kk & 3) * 32);
            umma_bf16(d_tmem, adesc, bdesc, kIdescR, (part > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&rbempty[s]);
        }
        umma_commit(&rfull[ab]);
        ++rit;
        if (++r_rt == p.n_rt) {
          r_rt = 0;
          ++r_gl;
        }
        return true;
      };
      for (int gl = 0; gl < ng && ok; ++gl) {
        // the query's router pairs must all be issued before its scoring
        while (ok && r_gl <= gl) router_pair(true);
        if (!ok) break;
        const int qb = gl & 1;
        if (!mbar_wait(&qfull[qb], static_cast<uint32_t>((gl >> 1) & 1), p.err, abort)) break;
        const uint32_t q_addr = smem_u32(sq + qb * kFSQBytes);
        for (int64_t item = run_begin(gl); item < run_end(gl) && ok; ++item, ++acc, ++it) {
          // the next query's router pairs, as soon as their operands are in
          while (ok && r_gl == gl + 1 && r_gl < ng && router_pair(false)) {
          }
          const int ta = static_cast<int>(acc & 1);
          if (!mbar_wait(&tempty[ta], static_cast<uint32_t>(((acc >> 1) & 1) ^ 1), p.err, abort)) { ok = false; break; }
          const int s = static_cast<int>(it % kFStages);
          if (!mbar_wait(&full[s], static_cast<uint32_t>((it / kFStages) & 1), p.err, abort)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(ring + s * kFTileBytes);
          const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(2 * NR + ta * kFHP);
#pragma unroll
          for (int kk = 0; kk < kD / 16; ++kk) {
            const uint64_t adesc = sw128_kmajor_desc(a_addr + (kk >> 2) * (kFTileM * 128) + (kk & 3) * 32);
            const uint64_t bdesc = sw128_kmajor_desc(q_addr + (kk >> 2) * (kFHP * 128) + (kk & 3) * 32);
            umma_bf16(d_tmem, adesc, bdesc, kIdescS, kk > 0 ? 1u : 0u);
          }
          umma_commit(&empty[s]);
          umma_commit(&tfull[ta]);
        }
        umma_commit(&qempty[qb]);
      }
      umma_commit(done);
      mbar_wait(done, 0, p.err);
    }
    __syncwarp();
  } else if (warp >= kFRouteWarp0) {
    // ------------------------------------------------------------ router epilogue (warps 4-7)
    const int rtid = tid - kFRouteWarp0 * 32, rwarp = rtid >> 5;
    const uint32_t t_lane = tmem_base + (static_cast<uint32_t>(rwarp * 32) << 16);
    int64_t rit = 0;
    bool skip = false;
    for (int gl = 0; gl < ng; ++gl) {
      const int g = g0 + gl;
      const int nvis = f_visible_blocks(p, g);
      const float* wrow = p.w + static_cast<int64_t>(g) * p.H;
      const float wmine = rtid < p.H ? wrow[rtid] : 0.f;
      for (int hh = rtid; hh < kFMaxNR; hh += kFEpiThreads) imp[hh] = 0.f;
      for (int rt = 0; rt < p.n_rt; ++rt, ++rit) {
        const int ab = static_cast<int>(rit & 1);
        float v[NR];
        const bool got = !skip && mbar_wait(&rfull[ab], static_cast<uint32_t>((rit >> 1) & 1), p.err, abort);
        if (got) {
          tc_fence_after();
          uint32_t r[NR];
#pragma unroll
          for (int u = 0; u < NR / 16; ++u) tmem_ld16(t_lane + static_cast<uint32_t>(ab * NR + 16 * u), r + 16 * u);
          tmem_wait_ld();
          tc_fence_before();
          mbar_arrive(&rempty[ab]);
          const bool vis = rt * kFTileM + rwarp * 32 + lane < nvis;
#pragma unroll
          for (int i = 0; i < NR; ++i) v[i] = vis ? fmaxf(__uint_as_float(r[i]), 0.f) : 0.f;
        } else {
          skip = true;
#pragma unroll
          for (int i = 0; i < NR; ++i) v[i] = 0.f;
        }
        f_lane_reduce<NR>(v, lane);
        const int h0 = f_lane_head0<NR>(lane);
        if (NR >= 32 || (lane & 1) == 0) {
#pragma unroll
          for (int i = 0; i < f_lane_heads<NR>(); ++i) red[rwarp * kFMaxNR + h0 + i] = v[i];
        }
        named_bar_sync(2, kFEpiThreads);
        if (rtid < p.H) imp[rtid] += ((red[rtid] + red[kFMaxNR + rtid]) + red[2 * kFMaxNR + rtid]) + red[3 * kFMaxNR + rtid];
        named_bar_sync(2, kFEpiThreads);
      }
      // importance and top-h (rank by counting; ties to the lower head)
      if (rtid < p.H) imp[rtid] = wmine * imp[rtid];
      named_bar_sync(2, kFEpiThreads);
      bool sel = false;
      if (rtid < p.H) {
        const float kNegInf = -__int_as_float(0x7f800000);
        float x = imp[rtid];
        x = x == x ? x : kNegInf;
        int rk = 0;
        for (int j = 0; j < p.H; ++j) {
          float y = imp[j];
          y = y == y ? y : kNegInf;
          rk += (y > x || (y == x && j < rtid)) ? 1 : 0;
        }
        sel = rk < p.h;
      }
      const unsigned bal = __ballot_sync(0xffffffffu, sel);
      if (lane == 0) misc[rwarp] = static_cast<uint32_t>(__popc(bal));
      if (rtid < kFHP) heads_r[rtid] = -1;
      named_bar_sync(2, kFEpiThreads);
      int before = 0;
      for (int w2 = 0; w2 < rwarp; ++w2) before += static_cast<int>(misc[w2]);
      const int pos = before + __popc(bal & ((1u << lane) - 1u));
      if (sel && pos < p.h) heads_r[pos] = rtid;
      // the CTA that holds the query's first tile reports heads and importances
      if (i0 <= static_cast<int64_t>(g) * tpg && !skip) {
        if (sel && pos < p.h) p.heads[static_cast<int64_t>(g) * p.h + pos] = rtid;
        if (p.importance && rtid < p.H) p.importance[static_cast<int64_t>(g) * p.H + rtid] = imp[rtid];
      }
      named_bar_sync(2, kFEpiThreads);
      // routed rows and weights into buffer gl & 1 once the query two back is done with it
      const int qb = gl & 1;
      if (gl >= 2 && !skip) {
        const uint32_t ph = static_cast<uint32_t>(((gl >> 1) - 1) & 1);
        if (!mbar_wait(&qempty[qb], ph, p.err, abort) || !mbar_wait(&wempty[qb], ph, p.err, abort)) skip = true;
      }
      if (!skip && !mbar_wait(qa_full, gl & 1, p.err, abort)) skip = true;
      uint8_t* sqb = sq + qb * kFSQBytes;
      for (int x = rtid; x < kFHP * 16; x += kFEpiThreads) {
        const int col = x >> 4, ch = x & 15;
        const int head = heads_r[col];
        uint4 val = make_uint4(0u, 0u, 0u, 0u);
        if (head >= 0) val = *reinterpret_cast<const uint4*>(qall + sw128_tile_offset(NR, head, ch));
        *reinterpret_cast<uint4*>(sqb + sw128_tile_offset(kFHP, col, ch)) = val;
      }
      if (rtid < kFHP) {
        const int head = heads_r[rtid];
        w_s[qb * kFHP + rtid] = head >= 0 ? wrow[head] : 0.f;   // padding columns: weight 0
      }
      fence_proxy_async_smem();
      mbar_arrive(qa_empty);     // the query rows may be replaced by the next query's
      mbar_arrive(&qfull[qb]);
      named_bar_sync(2, kFEpiThreads);   // heads_r / imp / red are reused by the next query
    }
  } else {
    // ------------------------------------------------------------ scoring epilogue (warps 0-3)
    const uint32_t t_lane = tmem_base + (static_cast<uint32_t>(warp * 32) << 16);
    int64_t acc = 0;
    bool skip = false;
    const int r = warp * 32 + lane;
    for (int gl = 0; gl < ng; ++gl) {
      const int g = g0 + gl;
      const int qb = gl & 1;
      float wv[kFHP];
      if (!skip && !mbar_wait(&qfull[qb], static_cast<uint32_t>((gl >> 1) & 1), p.err, abort)) skip = true;
#pragma unroll
      for (int i = 0; i < kFHP; ++i) wv[i] = w_s[qb * kFHP + i];
      mbar_arrive(&wempty[qb]);
      const int plen = f_valid_len(p, g);
      float* rowp = p.scores + static_cast<int64_t>(g) * p.row_stride;
      for (int64_t item = run_begin(gl); item < run_end(gl); ++item, ++acc) {
        const int ta = static_cast<int>(acc & 1);
        const bool ok = !skip && mbar_wait(&tfull[ta], static_cast<uint32_t>((acc >> 1) & 1), p.err, abort);
        if (!__all_sync(0xffffffffu, ok)) {   // warp-uniform, for the warp-wide TMEM load
          skip = true;
          continue;
        }
        tc_fence_after();
        uint32_t v[kFHP];
        tmem_ld16(t_lane + static_cast<uint32_t>(2 * NR + ta * kFHP), v);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(&tempty[ta]);
        float sacc = 0.f;
#pragma unroll
        for (int i = 0; i < kFHP; ++i) sacc = fmaf(wv[i], fmaxf(__uint_as_float(v[i]), 0.f), sacc);
        const int j = static_cast<int>(item - static_cast<int64_t>(g) * tpg);
        const int pos2 = j * kFTileM + r;
        if (pos2 < p.L) rowp[pos2] = pos2 < plen ? sacc : -__int_as_float(0x7f800000);   // stays in L2
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kFMmaWarp) tmem_dealloc(tmem_base, kFTmemCols);
}

}  // namespace

bool decode_fused_supported(int H, int h, int64_t L) {
  return H >= 1 && H <= kFMaxNR && h >= 1 && h <= kFHP && h <= H && L >= 1 && L <= kFMaxL;
}

cudaError_t launch_decode_fused(const DecodeArgs& a, cudaStream_t stream) {
  const int sms = device_sm_count();
  if (sms <= 0) return cudaErrorInvalidDevice;
  FusedParams p = {};
  p.q = a.q;
  p.w = a.w;
  p.seq_of = a.seq_of;
  p.prefix_len = a.prefix_len;
  p.T = a.T;
  p.H = a.H;
  p.h = a.h;
  p.L = a.L;
  p.B = a.B;
  p.M = static_cast<int>((a.L + a.B - 1) / a.B);
  p.n_rt = (p.M + kFTileM - 1) / kFTileM;
  p.key_seq_rows = a.key_seq_stride / kD;
  p.mean_seq_rows = a.means_seq_stride / kD;
  p.nkeyseq = a.nkeyseq;
  p.nmeanseq = a.nmeanseq;
  p.tpg = static_cast<int>((a.L + kFTileM - 1) / kFTileM);
  p.n_items = static_cast<int64_t>(a.T) * p.tpg;
  p.heads = a.heads;
  p.importance = a.importance;
  p.scores = a.scores;
  p.row_stride = a.row_stride;
  p.err = a.err;
  const int64_t grid = std::min<int64_t>(p.n_items, sms);

  // tensor maps: keys (128-row tiles as 64-row boxes, 128-byte swizzle), the
  // bf16 hi / lo block means (same layout), the query rows (box of H rows)
  CUtensorMap kmap, hmap, lmap, qmap;
  const uint64_t krows = static_cast<uint64_t>(a.nkeyseq - 1) * static_cast<uint64_t>(p.key_seq_rows) + a.L;
  const uint64_t mrows = static_cast<uint64_t>(a.nmeanseq - 1) * static_cast<uint64_t>(p.mean_seq_rows) + p.M;
  if (!encode_2d_map(&kmap, true, a.keys, kD, krows, kD * 2, 64, kTmaBoxRows, true) ||
      !encode_2d_map(&hmap, true, a.means_hi, kD, mrows, kD * 2, 64, kTmaBoxRows, true) ||
      !encode_2d_map(&lmap, true, a.means_lo, kD, mrows, kD * 2, 64, kTmaBoxRows, true) ||
      !encode_2d_map(&qmap, true, a.q, kD, static_cast<uint64_t>(a.T) * a.H, kD * 2, 64,
                     static_cast<uint32_t>(a.H), true))
    return cudaErrorInvalidValue;
  auto go = [&](auto kern) -> cudaError_t {
    cudaError_t e2 = ensure_dynamic_smem(reinterpret_cast<const void*>(kern), kFSmemBytes);
    if (e2 != cudaSuccess) return e2;
    return launch_pdl(kern, dim3(static_cast<unsigned>(grid)), dim3(kFThreads), kFSmemBytes, stream, 0, kmap, hmap,
                      lmap, qmap, p);
  };
  const int nr = a.H <= 16 ? 16 : (a.H <= 32 ? 32 : 64);
  if (nr == 16) return go(decode_fused_kernel<16>);
  if (nr == 32) return go(decode_fused_kernel<32>);
  return go(decode_fused_kernel<64>);
}

}  // namespace misa
