// Indexer token scoring on the 5th-generation tensor cores (tcgen05 + TMEM).
//
//   S[t, s] = sum over active heads i of w[t, head_i] * ReLU(q[t, head_i] . k[s])
//
// "MISA: Mixture of Indexer Sparse Attention for Long-Context LLM Inference"
// (gist.science), Methodology: only the h active heads score every prefix
// token (the dense DSA indexer is the case h = H_I).  HISA explainer
// (zhichai.net), section 三, Stage 2: the same indexer restricted to candidate
// tokens.
//
// One persistent CTA per SM.  The work is a list of items (column group g, key
// tile j): the 128 keys of tile j form the MMA's M dimension (A operand,
// K-major, 128-byte swizzled, one 32 KB shared-memory stage), and the group's
// (query, active head) query rows form N (B operand, resident in shared memory
// while the CTA works on that group).  The fp32 accumulator D[128 x N] lives in
// TMEM (two buffers, so the MMA of tile j+1 overlaps the epilogue of tile j).
// The epilogue reads D with tcgen05.ld (one TMEM lane = one key), applies ReLU,
// multiplies by the head weight and sums the heads of each query in ascending
// head order, and writes fp32 scores (coalesced, -inf past the prefix).
//
// Warp roles (EW epilogue warps per TMEM lane quarter: 1 when a group is one
// query, 4 when 32 queries share a tile of N = 256 columns):
//   warps 0 .. 4EW-1   epilogue (warp w reads TMEM lane quarter w % 4 and
//                      owns columns [(w / 4) N / EW, (w / 4 + 1) N / EW))
//   warp  4EW          TMEM allocation + single-thread MMA issue
//   warps 4EW+1 .. +4  producers.  Contiguous keys: warp 5 (one thread) streams the key
//              tiles by TMA from the first cycle while warps 6-8 stage the
//              group's query rows.  Candidate keys: all 128 threads stage the
//              query rows, then gather candidate rows with 16-byte cp.async.
// Every mbarrier wait is bounded; a wait that gives up records
// MISA_DEVERR_TIMEOUT, the role stops, in-flight copies and MMAs are waited for
// (bounded), TMEM is freed and the kernel returns.
#include <algorithm>
#include <cstring>

#include "launch.h"
#include "misa_device.cuh"

namespace misa {

namespace {

constexpr int kTileM = 128;                      // keys per tile (MMA M)
constexpr int kATileBytes = kTileM * kD * 2;     // 32 KB
constexpr int kProdThreads = 128;
#ifndef MISA_GATHER_LAG
#define MISA_GATHER_LAG 2
#endif
constexpr int kGatherLag = MISA_GATHER_LAG;  // tiles of gathered rows in flight per producer thread
#ifndef MISA_SHARED_EPI_WARPS
#define MISA_SHARED_EPI_WARPS 4
#endif
constexpr int kSharedEW = MISA_SHARED_EPI_WARPS;  // epilogue warps per lane quarter, shared-cache groups
#ifndef MISA_DECODE_CTAS
#define MISA_DECODE_CTAS 2
#endif
#ifndef MISA_DECODE_STAGES
#define MISA_DECODE_STAGES 3
#endif
constexpr int kDecodeCtas = MISA_DECODE_CTAS;
constexpr int kDecodeStages = MISA_DECODE_STAGES;                    // cp.async groups left in flight per producer thread

struct ScoreParams {
  const uint16_t* q;
  const float* w;
  const uint16_t* keys;
  int64_t key_seq_stride;   // elements
  int64_t nkeyseq;
  const int32_t* seq_of;
  const int32_t* prefix_len;
  int T;
  int H;
  int64_t L;
  const int32_t* heads;     // NULL: all heads
  int h;                    // active heads per query (H when heads == NULL)
  int q_block;
  const int32_t* cand;      // NULL: contiguous keys
  int n_cand;
  const int32_t* blocks;    // block mode: [T][n_cand / run] chosen key blocks (-1 = empty), or NULL
  int run;                  // block mode: keys per block (64 or 128)
  int64_t n_blocks_seq;     // block mode: blocks per sequence (ids at or above are invalid)
  float* scores;
  int64_t row_stride;
  int n_groups;
  int tiles_per_group;
  int64_t n_items;
  uint32_t* err;
};

__host__ __device__ constexpr int pow2_at_least(int x, int lo) {
  int p = lo;
  while (p < x) p <<= 1;
  return p;
}

template <int HP, int QPG, int EW, bool kGather>
struct Cfg {
  static constexpr int N = HP * QPG;
  static_assert(N % 16 == 0 && N >= 16 && N <= 256, "MMA N must be a multiple of 16 in [16, 256]");
  // EW epilogue warps per TMEM lane quarter, each owning N / EW columns (whole queries)
  static_assert((N / EW) % HP == 0, "an epilogue warp must own whole queries");
  static constexpr int kEpiWarps = 4 * EW;
  static constexpr int kEpiThreads = 32 * kEpiWarps;
  static constexpr int kMmaWarp = kEpiWarps;
  static constexpr int kProdWarp0 = kEpiWarps + 1;
  static constexpr int kThreads = 32 * (kEpiWarps + 1 + kProdThreads / 32);
  static constexpr int kColsPerWarp = N / EW;
  // a CTA per query group streams its own key cache: kDecodeCtas CTAs per SM
  // with kDecodeStages 32 KB stages each; shared-cache groups: one CTA per SM
  static constexpr bool kPerQuery = (QPG == 1) && !kGather;
  static constexpr int kCtasPerSm = kPerQuery ? kDecodeCtas : 1;
  static constexpr int kStages = kPerQuery ? kDecodeStages : (N >= 256 ? 4 : (N >= 128 ? 5 : 6));
  static constexpr int kQBytes = N * kD * 2;
  static constexpr int kTmemCols = pow2_at_least(2 * N, 32);
  static constexpr uint32_t kIdesc = idesc_bf16_f32(kTileM, N);
  // shared memory map (offsets from a 1024-byte aligned base)
  static constexpr int kOffA = 0;
  static constexpr int kOffQ = kStages * kATileBytes;
  static constexpr int kOffBar = kOffQ + kQBytes;
  static constexpr int kNumBars = 2 * kStages + 2 + 2 + 3;
  static constexpr int kOffTmemSlot = kOffBar + kNumBars * 8;
  static constexpr int kOffAbort = kOffTmemSlot + 4;
  static constexpr int kOffW = (kOffAbort + 4 + 15) / 16 * 16;
  static constexpr int kOffPlen = kOffW + N * 4;
  static constexpr int kOffRow = kOffPlen + (QPG * 4 + 7) / 8 * 8;
  static constexpr int kSmemBytes = kOffRow + QPG * 8 + 1024;  // + alignment slack
};

__device__ __forceinline__ void item_range(int64_t n_items, int64_t& i0, int64_t& i1) {
  const int64_t c = blockIdx.x, g = gridDim.x;
  i0 = n_items * c / g;
  i1 = n_items * (c + 1) / g;
}

// Stage the query rows of column group g into the B operand (K-major, 128-byte
// swizzled): column c = ql * HP + i holds q[t][head_i] of query t = g*QPG + ql,
// or zeros for padding columns.  Threads [0, nthreads) of the caller share it.
template <int HP, int QPG>
__device__ __forceinline__ void stage_query_rows(const ScoreParams& p, int g, uint8_t* sQ, int tid, int nthreads) {
  constexpr int N = HP * QPG;
  for (int x = tid; x < N * 16; x += nthreads) {
    const int c = x >> 4, ch = x & 15;
    const int ql = c / HP, i = c % HP;
    const int t = g * QPG + ql;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (t < p.T && i < p.h) {
      int head = i;
      if (p.heads) {
        head = p.heads[static_cast<int64_t>(t / p.q_block) * p.h + i];
        if (head < 0 || head >= p.H) {
          record_error(p.err, MISA_DEVERR_BAD_HEAD);
          head = -1;
        }
      }
      if (head >= 0)
        v = __ldg(reinterpret_cast<const uint4*>(p.q + (static_cast<int64_t>(t) * p.H + head) * kD + ch * 8));
    }
    *reinterpret_cast<uint4*>(sQ + sw128_tile_offset(N, c, ch)) = v;
  }
}

template <int HP, int QPG, int EW, bool kGather>
__global__ void __launch_bounds__(Cfg<HP, QPG, EW, kGather>::kThreads, Cfg<HP, QPG, EW, kGather>::kCtasPerSm)
score_kernel(const __grid_constant__ CUtensorMap tmap, const ScoreParams p) {
  using C = Cfg<HP, QPG, EW, kGather>;
  constexpr int kEpiThreads = C::kEpiThreads;
  constexpr int kMmaWarp = C::kMmaWarp;
  constexpr int kProdWarp0 = C::kProdWarp0;
  constexpr int N = C::N;
  constexpr int S = C::kStages;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem + C::kOffA;
  uint8_t* sQ = smem + C::kOffQ;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* full = bars;              // [S]  key tile landed
  uint64_t* empty = bars + S;         // [S]  MMAs reading the tile finished
  uint64_t* tfull = bars + 2 * S;     // [2]  accumulator ready
  uint64_t* tempty = bars + 2 * S + 2;  // [2]  accumulator drained
  uint64_t* qfull = bars + 2 * S + 4;   // group query rows staged
  uint64_t* qempty = bars + 2 * S + 5;  // MMAs of the group finished
  uint64_t* done = bars + 2 * S + 6;    // all MMAs of this CTA finished
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffTmemSlot);
  volatile uint32_t* abort = reinterpret_cast<volatile uint32_t*>(smem + C::kOffAbort);
  float* w_s = reinterpret_cast<float*>(smem + C::kOffW);
  int32_t* plen_s = reinterpret_cast<int32_t*>(smem + C::kOffPlen);   // visible keys of each group query
  float** rowp_s = reinterpret_cast<float**>(smem + C::kOffRow);       // its score row (NULL past T)

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], kGather ? kProdThreads : 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], kEpiThreads);
    }
    mbar_init(qfull, kGather ? kProdThreads : kProdThreads - 32);
    mbar_init(qempty, 1);
    mbar_init(done, 1);
    *abort = 0u;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  if (!kGather && tid == kProdWarp0 * 32) tma_prefetch_desc(&tmap);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait_inputs();
  pdl_allow_next();

  int64_t i0, i1;
  item_range(p.n_items, i0, i1);
  const int tpg = p.tiles_per_group;

  if (warp >= kProdWarp0) {
    // ------------------------------------------------------------ producers
    const int pt = tid - kProdWarp0 * 32;
    if (!kGather) {
      if (warp == kProdWarp0) {
        // one thread streams the key tiles by TMA; it starts at once and never
        // waits for the query rows
        if (lane == 0) {
          // a per-query cache is streamed once (evict first); a shared cache is
          // read by every column group (keep it in L2)
          const uint64_t policy = QPG == 1 ? l2_evict_first_policy() : l2_evict_last_policy();
          int64_t it = 0;
          int cur_g = -1;
          int64_t seq_row0 = 0;
          for (int64_t item = i0; item < i1; ++item) {
            const int g = static_cast<int>(item / tpg);
            const int j = static_cast<int>(item - static_cast<int64_t>(g) * tpg);
            if (g != cur_g) {
              int64_t seq = 0;
              if (QPG == 1) {
                seq = p.seq_of[g];
                if (seq < 0 || seq >= p.nkeyseq) {
                  record_error(p.err, MISA_DEVERR_BAD_SEQ);
                  seq = 0;
                }
              }
              seq_row0 = seq * (p.key_seq_stride / kD);
              cur_g = g;
            }
            const int s = static_cast<int>(it % S);
            const uint32_t ph = static_cast<uint32_t>((it / S) & 1);
            if (!mbar_wait(&empty[s], ph ^ 1u, p.err, abort)) break;
            uint8_t* dst = sA + s * kATileBytes;
            if (p.blocks == nullptr) {
              mbar_arrive_expect_tx(&full[s], kATileBytes);
              const int y = static_cast<int>(seq_row0 + static_cast<int64_t>(j) * kTileM);
#pragma unroll
              for (int r0 = 0; r0 < kTileM; r0 += kTmaBoxRows) {
                tma_load_2d_hint(dst + r0 * 128, &tmap, &full[s], 0, y + r0, policy);
                tma_load_2d_hint(dst + kATileBytes / 2 + r0 * 128, &tmap, &full[s], 64, y + r0, policy);
              }
            } else {
              // block mode: the 64-row box at candidate slot c holds keys
              // blocks[c / run] * run + c % run ...; a box of an empty block slot
              // (or past the list) is not loaded (its rows are masked)
              int yb[kTileM / kTmaBoxRows];
              uint32_t bytes = 0;
#pragma unroll
              for (int b2 = 0; b2 < kTileM / kTmaBoxRows; ++b2) {
                const int slot = j * kTileM + b2 * kTmaBoxRows;
                int64_t blk = -1;
                if (slot < p.n_cand) blk = p.blocks[static_cast<int64_t>(g) * (p.n_cand / p.run) + slot / p.run];
                if (blk >= p.n_blocks_seq) {
                  record_error(p.err, MISA_DEVERR_BAD_INDEX);
                  blk = -1;
                }
                yb[b2] = blk >= 0 ? static_cast<int>(seq_row0 + blk * p.run + slot % p.run) : -1;
                if (yb[b2] >= 0) bytes += kATileBytes / (kTileM / kTmaBoxRows);
              }
              mbar_arrive_expect_tx(&full[s], bytes);
#pragma unroll
              for (int b2 = 0; b2 < kTileM / kTmaBoxRows; ++b2) {
                if (yb[b2] < 0) continue;
                const int r0 = b2 * kTmaBoxRows;
                tma_load_2d_hint(dst + r0 * 128, &tmap, &full[s], 0, yb[b2], policy);
                tma_load_2d_hint(dst + kATileBytes / 2 + r0 * 128, &tmap, &full[s], 64, yb[b2], policy);
              }
            }
            ++it;
          }
          // make sure no TMA write into shared memory is still in flight
          const int64_t first = it > S ? it - S : 0;
          for (int64_t k = first; k < it; ++k) mbar_wait(&full[k % S], static_cast<uint32_t>((k / S) & 1), p.err);
        }
      } else {
        // the other three warps stage each group's query rows
        const int g0 = static_cast<int>(i0 / tpg);
        const int g1 = static_cast<int>((i1 - 1) / tpg);
        for (int g = g0, groups = 0; g <= g1; ++g, ++groups) {
          if (groups > 0 && !mbar_wait(qempty, (groups - 1) & 1, p.err, abort)) break;
          stage_query_rows<HP, QPG>(p, g, sQ, pt - 32, kProdThreads - 32);
          fence_proxy_async_smem();
          mbar_arrive(qfull);
        }
      }
    } else {
      // gather mode: all 128 producer threads stage the query rows, then
      // gather the candidate key rows with 16-byte cp.async.  Thread pt copies
      // chunk pt % 16 of rows pt / 16 + 8 i (i < 16) of every tile; the
      // candidate ids of the next tile are loaded one tile ahead, so a tile's
      // copies are issued without waiting for its ids.
      int64_t it = 0;
      int groups = 0;
      int cur_g = -1;
      bool ok = true;
      int64_t seq_row0 = 0;
      int64_t pending_from = 0;  // first iteration not yet signalled
      constexpr int kRowsPerThread = kTileM * 16 / kProdThreads;  // 16
      int32_t next_ids[kRowsPerThread];
      auto load_ids = [&](int64_t item2, int32_t (&dst)[kRowsPerThread]) {
        const int g2 = static_cast<int>(item2 / tpg);
        const int j2 = static_cast<int>(item2 - static_cast<int64_t>(g2) * tpg);
        const int32_t* crow = p.cand + static_cast<int64_t>(g2) * p.n_cand;
#pragma unroll
        for (int i = 0; i < kRowsPerThread; ++i) {
          const int64_t pos = static_cast<int64_t>(j2) * kTileM + (pt >> 4) + 8 * i;
          dst[i] = pos < p.n_cand ? __ldg(crow + pos) : -1;
        }
      };
      if (i0 < i1) load_ids(i0, next_ids);
      for (int64_t item = i0; item < i1 && ok; ++item) {
        const int g = static_cast<int>(item / tpg);
        const int j = static_cast<int>(item - static_cast<int64_t>(g) * tpg);
        if (g != cur_g) {
          // signal every outstanding stage before waiting on the MMA
          cp_async_wait_group<0>();
          fence_proxy_async_smem();
          for (; pending_from < it; ++pending_from) mbar_arrive(&full[pending_from % S]);
          if (groups > 0 && !mbar_wait(qempty, (groups - 1) & 1, p.err, abort)) { ok = false; break; }
          stage_query_rows<HP, QPG>(p, g, sQ, pt, kProdThreads);
          fence_proxy_async_smem();
          mbar_arrive(qfull);
          ++groups;
          cur_g = g;
          int64_t seq = p.seq_of[g];
          if (seq < 0 || seq >= p.nkeyseq) {
            if (pt == 0) record_error(p.err, MISA_DEVERR_BAD_SEQ);
            seq = 0;
          }
          seq_row0 = seq * (p.key_seq_stride / kD);
        }
        int32_t ids[kRowsPerThread];
#pragma unroll
        for (int i = 0; i < kRowsPerThread; ++i) ids[i] = next_ids[i];
        if (item + 1 < i1) load_ids(item + 1, next_ids);
        (void)j;
        const int s = static_cast<int>(it % S);
        const uint32_t ph = static_cast<uint32_t>((it / S) & 1);
        if (!mbar_wait(&empty[s], ph ^ 1u, p.err, abort)) { ok = false; break; }
        uint8_t* dst = sA + s * kATileBytes;
        const int ch = pt & 15;
#pragma unroll
        for (int i = 0; i < kRowsPerThread; ++i) {
          const int r = (pt >> 4) + 8 * i;
          const int64_t id = ids[i];
          const bool valid = (id >= 0) && (id < p.L);
          const uint16_t* src = p.keys + (seq_row0 + (valid ? id : 0)) * kD + ch * 8;
          cp_async_16(dst + sw128_tile_offset(kTileM, r, ch), src, valid);
        }
        cp_async_commit();
        // keep at most kGatherLag tiles of copies in flight; signal the oldest
        if (it - pending_from >= kGatherLag) {
          cp_async_wait_group<kGatherLag>();
          fence_proxy_async_smem();
          mbar_arrive(&full[pending_from % S]);
          ++pending_from;
        }
        ++it;
      }
      cp_async_wait_group<0>();
      fence_proxy_async_smem();
      for (; pending_from < it; ++pending_from) mbar_arrive(&full[pending_from % S]);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      int64_t it = 0;
      int groups = 0;
      int cur_g = -1;
      const uint32_t q_addr = smem_u32(sQ);
      for (int64_t item = i0; item < i1; ++item) {
        const int g = static_cast<int>(item / tpg);
        if (g != cur_g) {
          if (!mbar_wait(qfull, groups & 1, p.err, abort)) break;
          ++groups;
          cur_g = g;
        }
        const int a = static_cast<int>(it & 1);
        const uint32_t aph = static_cast<uint32_t>((it >> 1) & 1);
        if (!mbar_wait(&tempty[a], aph ^ 1u, p.err, abort)) break;
        const int s = static_cast<int>(it % S);
        const uint32_t ph = static_cast<uint32_t>((it / S) & 1);
        if (!mbar_wait(&full[s], ph, p.err, abort)) break;
        tc_fence_after();
        const uint32_t a_addr = smem_u32(sA + s * kATileBytes);
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(a * N);
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint64_t adesc = sw128_kmajor_desc(a_addr + (kk >> 2) * (kTileM * 128) + (kk & 3) * 32);
          const uint64_t bdesc = sw128_kmajor_desc(q_addr + (kk >> 2) * (N * 128) + (kk & 3) * 32);
          umma_bf16(d_tmem, adesc, bdesc, C::kIdesc, kk > 0 ? 1u : 0u);
        }
        umma_commit(&empty[s]);
        const bool group_ends = (item + 1 == i1) || (static_cast<int>((item + 1) / tpg) != g);
        if (group_ends) umma_commit(qempty);
        umma_commit(&tfull[a]);
        ++it;
      }
      umma_commit(done);
      mbar_wait(done, 0, p.err);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;          // TMEM lane quarter this warp may read
    const int cslice = warp >> 2;          // which N / EW columns it owns
    constexpr int NW = C::kColsPerWarp;
    const int col0 = cslice * NW;
    const int ql0 = col0 / HP;
    const int r = quarter * 32 + lane;     // TMEM lane = key row of the tile
    const uint32_t t_lane = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
    // After a wait gives up the loop keeps running without work ("skip"), so
    // every epilogue thread still reaches every named barrier.
    int64_t it = 0;
    int cur_g = -1;
    bool skip = false;
    for (int64_t item = i0; item < i1; ++item) {
      const int g = static_cast<int>(item / tpg);
      const int j = static_cast<int>(item - static_cast<int64_t>(g) * tpg);
      if (g != cur_g) {
        named_bar_sync(1, kEpiThreads);
        for (int c = tid; c < N; c += kEpiThreads) {
          const int ql = c / HP, i = c % HP;
          const int t = g * QPG + ql;
          float wv = 0.f;
          if (t < p.T && i < p.h) {
            int head = i;
            if (p.heads) head = p.heads[static_cast<int64_t>(t / p.q_block) * p.h + i];
            if (head >= 0 && head < p.H) wv = p.w[static_cast<int64_t>(t) * p.H + head];
          }
          w_s[c] = wv;
        }
        for (int ql = tid; ql < QPG; ql += kEpiThreads) {
          const int t = g * QPG + ql;
          int64_t pl = 0;
          if (t < p.T) {
            pl = p.prefix_len[t];
            if (pl > p.L) pl = p.L;
            if (pl < 0) pl = 0;
          }
          plen_s[ql] = static_cast<int32_t>(pl);
          rowp_s[ql] = (t < p.T) ? p.scores + static_cast<int64_t>(t) * p.row_stride : nullptr;
        }
        named_bar_sync(1, kEpiThreads);
        cur_g = g;
      }
      const int a = static_cast<int>(it & 1);
      const uint32_t aph = static_cast<uint32_t>((it >> 1) & 1);
      if (skip || !mbar_wait(&tfull[a], aph, p.err, abort)) {
        skip = true;
        ++it;
        continue;
      }
      tc_fence_after();

      // which output slot this lane's key row maps to, and whether it is visible
      const int pos = j * kTileM + r;  // column of the score row (< 2^31)
      bool in_row;
      int key_id;
      if (kGather) {
        in_row = pos < p.n_cand;
        key_id = in_row ? p.cand[static_cast<int64_t>(g) * p.n_cand + pos] : -1;
      } else if (p.blocks != nullptr) {
        in_row = pos < p.n_cand;
        const int64_t blk = in_row ? p.blocks[static_cast<int64_t>(g) * (p.n_cand / p.run) + pos / p.run] : -1;
        key_id = (blk >= 0 && blk < p.n_blocks_seq) ? static_cast<int>(blk * p.run + pos % p.run) : -1;
      } else {
        in_row = pos < p.L;
        key_id = pos;
      }

      constexpr int kBatch = EW == 1 ? (NW < 64 ? NW : 64) : (NW < 32 ? NW : 32);
      const uint32_t t_acc = t_lane + static_cast<uint32_t>(a * N + col0);
      const float* wcol = w_s + col0;
      float sacc = 0.f;
#pragma unroll
      for (int c0 = 0; c0 < NW; c0 += kBatch) {
        uint32_t v[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch / 16; ++u)
          tmem_ld16(t_acc + static_cast<uint32_t>(c0 + 16 * u), v + 16 * u);
        tmem_wait_ld();
        if (c0 + kBatch == NW) {
          // this warp's part of the accumulator is read: hand it back
          tc_fence_before();
          mbar_arrive(&tempty[a]);
        }
#pragma unroll
        for (int jj = 0; jj < kBatch; ++jj) {
          const int col = c0 + jj;  // within this warp's columns
          const int i = col % HP;
          if (i == 0) sacc = 0.f;
          sacc = fmaf(wcol[col], fmaxf(__uint_as_float(v[jj]), 0.f), sacc);
          if (i == HP - 1) {
            const int ql = ql0 + col / HP;
            float* rp = rowp_s[ql];
            if (rp != nullptr && in_row) {
              // visible iff 0 <= key_id < prefix (one unsigned compare)
              const float val = static_cast<uint32_t>(key_id) < static_cast<uint32_t>(plen_s[ql])
                                    ? sacc
                                    : -__int_as_float(0x7f800000);
              if (QPG == 1) rp[pos] = val;     // re-read soon by the top-k: keep in L2
              else __stcs(rp + pos, val);      // large score matrix: stream past L2
            }
          }
        }
      }
      ++it;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem_base, C::kTmemCols);
}

template <int HP, int QPG, int EW, bool kGather>
cudaError_t launch_cfg(const CUtensorMap& tmap, const ScoreParams& p, int num_sms, cudaStream_t stream) {
  using C = Cfg<HP, QPG, EW, kGather>;
  auto kern = score_kernel<HP, QPG, EW, kGather>;
  cudaError_t e = ensure_dynamic_smem(reinterpret_cast<const void*>(kern), C::kSmemBytes);
  if (e != cudaSuccess) return e;
  const int per_sm = occupancy_blocks(reinterpret_cast<const void*>(kern), C::kThreads, C::kSmemBytes);
  int64_t grid = std::min<int64_t>(p.n_items, static_cast<int64_t>(num_sms) * std::max(1, std::min(per_sm, C::kCtasPerSm)));
  if (grid < 1) grid = 1;
  return launch_pdl(kern, dim3(static_cast<unsigned>(grid)), dim3(C::kThreads), C::kSmemBytes, stream, 0, tmap, p);
}

}  // namespace

int score_mode_hp(int h_eff, bool shared_groups) {
  const int hp = pow2_at_least(h_eff, 1);
  return shared_groups ? hp : std::max(16, hp);
}

cudaError_t launch_index_score(const CUtensorMap* tmap, const ScoreArgs& a, cudaStream_t stream) {
  const int num_sms = device_sm_count();
  if (num_sms <= 0) return cudaErrorInvalidDevice;

  const int h_eff = a.heads ? a.h : a.H;
  const bool gather = a.cand != nullptr;
  const bool shared_groups = !gather && a.blocks == nullptr && a.key_seq_stride == 0;
  const int hp = score_mode_hp(h_eff, shared_groups);
  const int qpg = shared_groups ? 256 / hp : 1;

  ScoreParams p;
  p.q = a.q;
  p.w = a.w;
  p.keys = a.keys;
  p.key_seq_stride = a.key_seq_stride;
  p.nkeyseq = a.nkeyseq;
  p.seq_of = a.seq_of;
  p.prefix_len = a.prefix_len;
  p.T = a.T;
  p.H = a.H;
  p.L = a.L;
  p.heads = a.heads;
  p.h = h_eff;
  p.q_block = a.q_block;
  p.cand = a.cand;
  p.n_cand = a.n_cand;
  p.blocks = a.blocks;
  p.run = a.run;
  p.n_blocks_seq = a.run > 0 ? (a.L + a.run - 1) / a.run : 0;
  p.scores = a.scores;
  p.row_stride = a.row_stride;
  p.err = a.err;
  if (gather || a.blocks) {
    p.n_groups = a.T;
    p.tiles_per_group = (a.n_cand + kTileM - 1) / kTileM;
  } else {
    p.n_groups = (a.T + qpg - 1) / qpg;
    p.tiles_per_group = static_cast<int>((a.L + kTileM - 1) / kTileM);
  }
  p.n_items = static_cast<int64_t>(p.n_groups) * p.tiles_per_group;
  if (p.n_items == 0) return cudaSuccess;

  CUtensorMap dummy;
  std::memset(&dummy, 0, sizeof(dummy));
  const CUtensorMap& tm = tmap ? *tmap : dummy;

  if (gather) {
    switch (hp) {
      case 16: return launch_cfg<16, 1, 1, true>(tm, p, num_sms, stream);
      case 32: return launch_cfg<32, 1, 1, true>(tm, p, num_sms, stream);
      case 64: return launch_cfg<64, 1, 1, true>(tm, p, num_sms, stream);
      case 128: return launch_cfg<128, 1, 1, true>(tm, p, num_sms, stream);
      default: return cudaErrorInvalidValue;
    }
  }
  if (!shared_groups) {
    switch (hp) {
      case 16: return launch_cfg<16, 1, 1, false>(tm, p, num_sms, stream);
      case 32: return launch_cfg<32, 1, 1, false>(tm, p, num_sms, stream);
      case 64: return launch_cfg<64, 1, 1, false>(tm, p, num_sms, stream);
      case 128: return launch_cfg<128, 1, 1, false>(tm, p, num_sms, stream);
      default: return cudaErrorInvalidValue;
    }
  }
  switch (hp) {
    case 1: return launch_cfg<1, 256, kSharedEW, false>(tm, p, num_sms, stream);
    case 2: return launch_cfg<2, 128, kSharedEW, false>(tm, p, num_sms, stream);
    case 4: return launch_cfg<4, 64, kSharedEW, false>(tm, p, num_sms, stream);
    case 8: return launch_cfg<8, 32, kSharedEW, false>(tm, p, num_sms, stream);
    case 16: return launch_cfg<16, 16, kSharedEW, false>(tm, p, num_sms, stream);
    case 32: return launch_cfg<32, 8, kSharedEW, false>(tm, p, num_sms, stream);
    case 64: return launch_cfg<64, 4, kSharedEW, false>(tm, p, num_sms, stream);
    case 128: return launch_cfg<128, 2, 2, false>(tm, p, num_sms, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace misa
