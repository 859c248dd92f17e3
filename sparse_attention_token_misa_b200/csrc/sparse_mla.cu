// Sparse attention over the indexer's selected tokens (the operator the
// indexer feeds), on the 5th-generation tensor cores.
//
// HISA explainer (zhichai.net), section 二 (DSA 的工作原理): after the indexer
// has picked k tokens per query, attention runs over those k tokens only;
// section 四 (Drop-in Replacement): that operator (Sparse MLA) takes the k token
// indices over the unchanged KV cache.  The KV cache holds one latent row of
// 576 bf16 per token shared by every query head (512 latent + 64 rotary): the
// keys are the whole row, the values its first 512 entries.
//
//   out[t, h] = sum_i p[h, i] * v_i / sum_i p[h, i],
//   p[h, i]   = exp(scale * q[t, h] . k_i - max_i(...)),   i over idx[t] (-1: empty)
//
// Work split: one CTA per (query t, chunk c of 256 index slots).  Inside a CTA,
// in order:
//  1. S = Q K^T on tcgen05: M = 128 query heads, N = 256 slots, K = 576 in 9
//     blocks of 64; the query block arrives by TMA, the 256 gathered key rows by
//     16-byte cp.async in the 128-byte-swizzled K-major layout; S in TMEM
//     columns [0, 256).
//  2. Exact softmax over the chunk: two epilogue threads per head h (one per
//     half of the slots) read their part of the S row twice from TMEM (max,
//     exchanged through shared memory, then exp2), round p to bf16, add the
//     rounded values into l and write p as the A operand of the next MMA
//     (K-major, swizzled) to shared memory.
//  3. O = P V: M = 128 heads, N = 512 value columns (two MMAs of 256), K = 256
//     slots in blocks of 32.  V is staged MN-major (each token's 512 values are
//     one row of eight 64-column swizzle atoms), so the gathered rows need no
//     transpose.  O takes all 512 TMEM columns; it overwrites S, which step 2
//     has finished reading.  The value gathers start as soon as the last QK
//     MMA has completed and overlap step 2.
//  4. O (unnormalised) and (m, l) of the chunk go to the workspace; a combine
//     kernel merges the chunks of each query (flash-decoding style) and writes
//     bf16 out and, optionally, the log-sum-exp.
//
// Roles (416 threads): warps 0-7 epilogue (warp w: TMEM lane quarter w % 4,
// slot / column half w / 4), warp 8 TMEM allocation + MMA issue, warps 9-12
// producers (thread 0 of them also issues the query TMA).  Waits are bounded
// and share a CTA-wide abort flag.
#include "launch.h"
#include "misa_device.cuh"

namespace misa {

namespace {

constexpr int kDqk = MISA_MLA_DQK;             // 576
constexpr int kDv = MISA_MLA_DV;               // 512
constexpr int kSlots = 256;                    // index slots per CTA (MMA N of S)
constexpr int kHM = 128;                       // MMA M: query heads
constexpr int kQKBlocks = kDqk / 64;           // 9 K blocks of 64
constexpr int kS1 = 3;                         // QK stages
constexpr int kQBlockBytes = kHM * 128;        // 16 KB: 128 heads x 64 bf16
constexpr int kKBlockBytes = kSlots * 128;     // 32 KB: 256 rows x 64 bf16
constexpr int kS1Bytes = kQBlockBytes + kKBlockBytes;
constexpr int kVTok = 32;                      // tokens per value stage
constexpr int kS3 = 4;                         // value stages
constexpr int kVAtomBytes = kVTok * 128;       // one 64-column atom of a value stage
constexpr int kVStageBytes = kVTok * kDv * 2;  // 32 KB
constexpr int kOffStage = 0;
constexpr int kStageRegion = kS1 * kS1Bytes;   // 144 KB (value stages reuse it)
static_assert(kS3 * kVStageBytes <= kStageRegion, "value stages must fit the QK stage region");
constexpr int kOffP = kOffStage + kStageRegion;
constexpr int kPBytes = kHM * kSlots * 2;      // 64 KB
constexpr int kOffIds = kOffP + kPBytes;
constexpr int kOffMask = kOffIds + kSlots * 4;   // [kSlots / 32] valid-slot bits
constexpr int kOffBar = kOffMask + (kSlots / 32) * 4;
constexpr int kNumBars = 2 * kS1 + 2 * kS3 + 4;
constexpr int kOffTmem = kOffBar + kNumBars * 8;
constexpr int kOffFlag = kOffTmem + 16;
constexpr int kOffRed = kOffFlag + 16;           // [2][kHM] per-half row maxima / sums
constexpr int kSmemBytes = kOffRed + 2 * kHM * 4 + 1024;
constexpr int kThreads = 416;
constexpr int kEpiThreads = 256;
constexpr int kMmaWarp = 8;
constexpr int kProdWarp0 = 9;
constexpr int kProdThreads = 128;
constexpr int kPitch = 132;                      // O staging row pitch (floats)
static_assert(2 * kHM * kPitch * 4 <= kStageRegion, "O staging must fit the stage region");
constexpr uint32_t kIdescS = idesc_bf16_f32(kHM, kSlots);
// P V: B (the values) is MN-major
constexpr uint32_t kIdescO = idesc_bf16_f32(kHM, 256) | (1u << 16);

// Descriptor of an MN-major operand in 128-byte swizzled atoms (64 columns x 8
// rows of K): 8-row groups 1024 bytes apart (SBO), 64-column atoms `lbo`
// bytes apart (LBO).
__device__ __forceinline__ uint64_t sw128_mnmajor_desc(uint32_t smem_addr, uint32_t lbo) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((smem_addr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>(1024u >> 4) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  d |= static_cast<uint64_t>(2u) << 61;
  return d;
}

struct MlaParams {
  const uint16_t* kv;
  int64_t kv_seq_stride;   // elements between sequences
  int64_t nseq, L;
  const int32_t* seq_of;
  int T, Hq;
  const int32_t* idx;
  int64_t idx_stride;
  int k, nch;
  float scale_log2;        // scale * log2(e)
  float* part_o;           // [T][nch][Hq][512]
  float* part_ml;          // [T][nch][Hq][2]: m (log2 units), l
  uint32_t* err;
};

__global__ void __launch_bounds__(kThreads, 1)
sparse_mla_kernel(const __grid_constant__ CUtensorMap q_map, const MlaParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sStage = smem + kOffStage;
  uint8_t* sP = smem + kOffP;
  int32_t* sIds = reinterpret_cast<int32_t*>(smem + kOffIds);
  uint32_t* sMask = reinterpret_cast<uint32_t*>(smem + kOffMask);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  uint64_t* full1 = bars;                    // [kS1] query block (TMA) + key rows (cp.async) landed
  uint64_t* empty1 = bars + kS1;             // [kS1] QK MMAs of the stage done
  uint64_t* full3 = bars + 2 * kS1;          // [kS3] value rows landed
  uint64_t* empty3 = bars + 2 * kS1 + kS3;   // [kS3] PV MMAs of the stage done
  uint64_t* sfull = bars + 2 * kS1 + 2 * kS3;  // S complete (and the QK stages free)
  uint64_t* pfull = sfull + 1;               // P written, S read
  uint64_t* ofull = sfull + 2;               // O complete
  uint64_t* done = sfull + 3;                // every MMA retired (teardown)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffTmem);
  volatile uint32_t* abort = reinterpret_cast<volatile uint32_t*>(smem + kOffFlag);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int t = static_cast<int>(blockIdx.x) / p.nch;
  const int c = static_cast<int>(blockIdx.x) - t * p.nch;
  if (tid == 0) {
    for (int s = 0; s < kS1; ++s) {
      mbar_init(&full1[s], kProdThreads + 1);
      mbar_init(&empty1[s], 1);
    }
    for (int s = 0; s < kS3; ++s) {
      mbar_init(&full3[s], kProdThreads);
      mbar_init(&empty3[s], 1);
    }
    mbar_init(sfull, 1);
    mbar_init(pfull, 1);
    mbar_init(ofull, 1);
    mbar_init(done, 1);
    *abort = 0u;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  if (tid == kProdWarp0 * 32) tma_prefetch_desc(&q_map);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait_inputs();
  pdl_allow_next();

  // slot ids of this chunk (-1: empty or out of range)
  for (int j = tid; j < kSlots; j += kThreads) {
    const int64_t slot = static_cast<int64_t>(c) * kSlots + j;
    int32_t id = -1;
    if (slot < p.k) {
      id = __ldg(p.idx + static_cast<int64_t>(t) * p.idx_stride + slot);
      if (id < -1 || id >= p.L) {
        record_error(p.err, MISA_DEVERR_BAD_INDEX);
        id = -1;
      }
    }
    sIds[j] = id;
  }
  __syncthreads();
  if (warp < kSlots / 32) {
    const unsigned bits = __ballot_sync(0xffffffffu, sIds[warp * 32 + lane] >= 0);
    if (lane == 0) sMask[warp] = bits;
  }
  __syncthreads();

  if (warp >= kProdWarp0) {
    // ------------------------------------------------------------ producers
    const int pt = tid - kProdWarp0 * 32;
    int64_t seq = p.seq_of[t];
    if (seq < 0 || seq >= p.nseq) {
      if (pt == 0) record_error(p.err, MISA_DEVERR_BAD_SEQ);
      seq = 0;
    }
    const uint16_t* kvs = p.kv + seq * p.kv_seq_stride;
    bool ok = true;
    // QK blocks: thread pt copies chunk pt % 8 of rows pt / 8 + 16 i (i < 16)
    {
      const int ch = pt & 7;
      int32_t ids[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) ids[i] = sIds[(pt >> 3) + 16 * i];
      int pending = 0;  // first block not yet signalled
      for (int kb = 0; kb < kQKBlocks; ++kb) {
        const int s = kb % kS1;
        const uint32_t ph = static_cast<uint32_t>((kb / kS1) & 1);
        if (!mbar_wait(&empty1[s], ph ^ 1u, p.err, abort)) { ok = false; break; }
        uint8_t* qdst = sStage + s * kS1Bytes;
        uint8_t* kdst = qdst + kQBlockBytes;
        if (pt == 0) {
          mbar_arrive_expect_tx(&full1[s], kQBlockBytes);
          tma_load_2d(qdst, &q_map, &full1[s], kb * 64, t * p.Hq);
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int r = (pt >> 3) + 16 * i;
          const bool valid = ids[i] >= 0;
          const uint16_t* src = kvs + static_cast<int64_t>(valid ? ids[i] : 0) * kDqk + kb * 64 + ch * 8;
          cp_async_16(kdst + r * 128 + ((ch ^ (r & 7)) << 4), src, valid);
        }
        cp_async_commit();
        if (kb - pending >= kS1 - 1) {
          cp_async_wait_group<kS1 - 1>();
          fence_proxy_async_smem();
          mbar_arrive(&full1[pending % kS1]);
          ++pending;
        }
      }
      cp_async_wait_group<0>();
      fence_proxy_async_smem();
      if (ok)
        for (; pending < kQKBlocks; ++pending) mbar_arrive(&full1[pending % kS1]);
    }
    // value blocks, once every QK MMA has completed (the stage region is free):
    // thread pt copies chunk pt % 64 (8 values) of tokens pt / 64 + 2 i (i < 16)
    if (ok && mbar_wait(sfull, 0, p.err, abort)) {
      const int ch = pt & 63;
      int pending = 0;
      constexpr int kVBlocks = kSlots / kVTok;  // 8
      for (int vb = 0; vb < kVBlocks; ++vb) {
        const int s = vb % kS3;
        const uint32_t ph = static_cast<uint32_t>((vb / kS3) & 1);
        if (!mbar_wait(&empty3[s], ph ^ 1u, p.err, abort)) { ok = false; break; }
        uint8_t* vdst = sStage + s * kVStageBytes;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int r = (pt >> 6) + 2 * i;
          const int32_t id = sIds[vb * kVTok + r];
          const bool valid = id >= 0;
          const uint16_t* src = kvs + static_cast<int64_t>(valid ? id : 0) * kDqk + ch * 8;
          cp_async_16(vdst + (ch >> 3) * kVAtomBytes + r * 128 + (((ch & 7) ^ (r & 7)) << 4), src, valid);
        }
        cp_async_commit();
        if (vb - pending >= kS3 - 1) {
          cp_async_wait_group<kS3 - 1>();
          fence_proxy_async_smem();
          mbar_arrive(&full3[pending % kS3]);
          ++pending;
        }
      }
      cp_async_wait_group<0>();
      fence_proxy_async_smem();
      if (ok)
        for (; pending < kVBlocks; ++pending) mbar_arrive(&full3[pending % kS3]);
    }
    cp_async_wait_group<0>();
    // no TMA write may still be in flight when the CTA exits
    if (pt == 0)
      for (int kb = kQKBlocks - kS1; kb < kQKBlocks; ++kb)
        mbar_wait(&full1[kb % kS1], static_cast<uint32_t>((kb / kS1) & 1), p.err);
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      const uint32_t s_tmem = tmem_base;
      bool ok = true;
      for (int kb = 0; kb < kQKBlocks && ok; ++kb) {
        const int s = kb % kS1;
        if (!mbar_wait(&full1[s], static_cast<uint32_t>((kb / kS1) & 1), p.err, abort)) { ok = false; break; }
        tc_fence_after();
        const uint32_t qa = smem_u32(sStage + s * kS1Bytes);
        const uint32_t ka = qa + kQBlockBytes;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_bf16(s_tmem, sw128_kmajor_desc(qa + kk * 32), sw128_kmajor_desc(ka + kk * 32), kIdescS,
                    (kb | kk) ? 1u : 0u);
        umma_commit(&empty1[s]);
      }
      if (ok) umma_commit(sfull);
      // P V once the softmax has written P and read S
      if (ok && mbar_wait(pfull, 0, p.err, abort)) {
        const uint32_t pa = smem_u32(sP);
        constexpr int kVBlocks = kSlots / kVTok;
        for (int vb = 0; vb < kVBlocks; ++vb) {
          const int s = vb % kS3;
          if (!mbar_wait(&full3[s], static_cast<uint32_t>((vb / kS3) & 1), p.err, abort)) { ok = false; break; }
          tc_fence_after();
          const uint32_t va = smem_u32(sStage + s * kVStageBytes);
#pragma unroll
          for (int kk = 0; kk < kVTok / 16; ++kk) {
            // P columns (slots) vb*32 + kk*16 .. +16: K block (vb*32)/64, 32-byte step inside it
            const int slot0 = vb * kVTok + kk * 16;
            const uint64_t adesc = sw128_kmajor_desc(pa + (slot0 >> 6) * (kHM * 128) + ((slot0 & 63) >> 3) * 16);
#pragma unroll
            for (int half = 0; half < 2; ++half) {
              const uint64_t bdesc = sw128_mnmajor_desc(va + half * 4 * kVAtomBytes + kk * 2048, kVAtomBytes);
              umma_bf16(tmem_base + half * 256, adesc, bdesc, kIdescO, (vb | kk) ? 1u : 0u);
            }
          }
          umma_commit(&empty3[s]);
        }
        if (ok) umma_commit(ofull);
      }
      umma_commit(done);
      mbar_wait(done, 0, p.err);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue (two threads per head row)
    const int quarter = warp & 3, half = warp >> 2;
    const int r = quarter * 32 + lane;  // head row
    const uint32_t t_lane = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
    const bool live = r < p.Hq;
    const float kNegInf = -__int_as_float(0x7f800000);
    float* sRed = reinterpret_cast<float*>(smem + kOffRed);
    // warp-uniform outcome of the wait: the TMEM loads below are warp-wide
    const bool ok = __all_sync(0xffffffffu, mbar_wait(sfull, 0, p.err, abort));
    const int cbeg = half * (kSlots / 2), cend = cbeg + kSlots / 2;
    float mx = kNegInf, l = 0.f;
    uint32_t v[16];
    if (ok) {
      tc_fence_after();
      for (int c0 = cbeg; c0 < cend; c0 += 16) {
        tmem_ld16(t_lane + c0, v);
        tmem_wait_ld();
        const uint32_t bits = sMask[c0 >> 5] >> (c0 & 31);
#pragma unroll
        for (int j = 0; j < 16; ++j)
          if ((bits >> j) & 1u) mx = fmaxf(mx, __uint_as_float(v[j]) * p.scale_log2);
      }
    }
    sRed[half * kHM + r] = mx;
    named_bar_sync(1, kEpiThreads);
    mx = fmaxf(sRed[r], sRed[kHM + r]);
    if (ok) {
      const bool any = mx != kNegInf;
      for (int c0 = cbeg; c0 < cend; c0 += 16) {
        tmem_ld16(t_lane + c0, v);
        tmem_wait_ld();
        const uint32_t bits = any ? sMask[c0 >> 5] >> (c0 & 31) : 0u;
        uint32_t w[8];
#pragma unroll
        for (int j = 0; j < 16; j += 2) {
          const float a = ((bits >> j) & 1u) ? exp2f(__uint_as_float(v[j]) * p.scale_log2 - mx) : 0.f;
          const float b = ((bits >> (j + 1)) & 1u) ? exp2f(__uint_as_float(v[j + 1]) * p.scale_log2 - mx) : 0.f;
          const __nv_bfloat16 ha = __float2bfloat16_rn(a), hb = __float2bfloat16_rn(b);
          l += __bfloat162float(ha) + __bfloat162float(hb);
          w[j >> 1] = static_cast<uint32_t>(__bfloat16_as_ushort(ha)) |
                      (static_cast<uint32_t>(__bfloat16_as_ushort(hb)) << 16);
        }
        // slots c0 .. c0+16 = two 16-byte chunks of K block c0 / 64
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int cc = ((c0 & 63) >> 3) + u;
          *reinterpret_cast<uint4*>(sP + (c0 >> 6) * (kHM * 128) + r * 128 + ((cc ^ (r & 7)) << 4)) =
              make_uint4(w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
        }
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    named_bar_sync(1, kEpiThreads);  // P complete, S read, every maximum read
    if (ok && warp == 0 && lane == 0) mbar_arrive(pfull);
    sRed[half * kHM + r] = l;
    named_bar_sync(1, kEpiThreads);
    if (half == 0 && live) {
      const int64_t prow = (static_cast<int64_t>(t) * p.nch + c) * p.Hq + r;
      p.part_ml[prow * 2] = mx;
      p.part_ml[prow * 2 + 1] = sRed[r] + sRed[kHM + r];
    }
    // O by quarters of 128 columns (half h: quarters 2h, 2h + 1) through the
    // (now idle) stage region, so that each row leaves as one coalesced
    // 512-byte store: thread r writes its row quarter at pitch 132 floats (4
    // store wavefronts per warp, the minimum), then the half's warp q copies
    // rows q, q + 4, ...
    const bool ok_o = __all_sync(0xffffffffu, ok && mbar_wait(ofull, 0, p.err, abort));
    if (ok_o) tc_fence_after();
    float* stg = reinterpret_cast<float*>(sStage) + half * (kHM * kPitch);
    for (int qq = 0; qq < 2; ++qq) {
      const int q4 = half * 2 + qq;
      if (ok_o) {
        for (int u = 0; u < 8; ++u) {
          tmem_ld16(t_lane + q4 * 128 + u * 16, v);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 16; j += 4)
            *reinterpret_cast<float4*>(stg + r * kPitch + u * 16 + j) = make_float4(
                __uint_as_float(v[j]), __uint_as_float(v[j + 1]), __uint_as_float(v[j + 2]), __uint_as_float(v[j + 3]));
        }
      }
      named_bar_sync(2 + half, kEpiThreads / 2);
      if (ok_o) {
        for (int rr = quarter; rr < p.Hq; rr += 4) {
          const float4 x = *reinterpret_cast<const float4*>(stg + rr * kPitch + lane * 4);
          const int64_t orow = (static_cast<int64_t>(t) * p.nch + c) * p.Hq + rr;
          *reinterpret_cast<float4*>(p.part_o + orow * kDv + q4 * 128 + lane * 4) = x;
        }
      }
      named_bar_sync(2 + half, kEpiThreads / 2);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem_base, 512);
}

// out[t, h] = sum_c 2^(m_c - m) O_c / sum_c 2^(m_c - m) l_c, m = max_c m_c; one
// CTA of 128 threads per (t, h), 4 value columns per thread.  The chunk
// statistics are read by one thread each, the weights and the denominator are
// formed in chunk order (deterministic), and the chunk rows are then loaded
// four at a time.
constexpr int kMaxChunks = (MISA_MAX_TOPK + kSlots - 1) / kSlots;  // 64
__global__ void __launch_bounds__(128)
sparse_mla_combine_kernel(const float* __restrict__ part_o, const float* __restrict__ part_ml, int T, int Hq,
                          int nch, uint16_t* __restrict__ out, float* __restrict__ lse) {
  __shared__ float s_m[kMaxChunks], s_w[kMaxChunks];
  __shared__ float s_den;
  pdl_wait_inputs();
  pdl_allow_next();
  const int th = static_cast<int>(blockIdx.x);
  const int t = th / Hq, h = th - t * Hq;
  const int tid = threadIdx.x;
  const float kNegInf = -__int_as_float(0x7f800000);
  const int64_t row0 = static_cast<int64_t>(t) * nch * Hq + h;  // chunk c: row0 + c * Hq
  float lc = 0.f;
  if (tid < nch) {
    s_m[tid] = part_ml[(row0 + static_cast<int64_t>(tid) * Hq) * 2];
    lc = part_ml[(row0 + static_cast<int64_t>(tid) * Hq) * 2 + 1];
  }
  __syncthreads();
  float m = kNegInf;
  for (int c = 0; c < nch; ++c) m = fmaxf(m, s_m[c]);
  if (tid < nch) s_w[tid] = (m == kNegInf || s_m[tid] == kNegInf) ? 0.f : exp2f(s_m[tid] - m);
  __syncthreads();
  if (tid < nch) s_m[tid] = s_w[tid] * lc;  // weighted sums, reusing s_m
  __syncthreads();
  if (tid == 0) {
    float den = 0.f;
    for (int c = 0; c < nch; ++c) den += s_m[c];
    s_den = den;
  }
  __syncthreads();
  const float den = s_den;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  const float4* base = reinterpret_cast<const float4*>(part_o + row0 * kDv) + tid;
  const int64_t cstride = static_cast<int64_t>(Hq) * kDv / 4;  // float4s between chunks
  int c = 0;
  for (; c + 4 <= nch; c += 4) {
    float4 o[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) o[u] = s_w[c + u] != 0.f ? __ldcs(base + (c + u) * cstride) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const float wc = s_w[c + u];
      acc.x += wc * o[u].x;
      acc.y += wc * o[u].y;
      acc.z += wc * o[u].z;
      acc.w += wc * o[u].w;
    }
  }
  for (; c < nch; ++c) {
    const float wc = s_w[c];
    if (wc == 0.f) continue;
    const float4 o = __ldcs(base + c * cstride);
    acc.x += wc * o.x;
    acc.y += wc * o.y;
    acc.z += wc * o.z;
    acc.w += wc * o.w;
  }
  const float inv = den > 0.f ? 1.0f / den : 0.f;
  const __nv_bfloat16 a = __float2bfloat16_rn(acc.x * inv), b = __float2bfloat16_rn(acc.y * inv);
  const __nv_bfloat16 c2 = __float2bfloat16_rn(acc.z * inv), d = __float2bfloat16_rn(acc.w * inv);
  uint2 packed;
  packed.x = static_cast<uint32_t>(__bfloat16_as_ushort(a)) | (static_cast<uint32_t>(__bfloat16_as_ushort(b)) << 16);
  packed.y = static_cast<uint32_t>(__bfloat16_as_ushort(c2)) | (static_cast<uint32_t>(__bfloat16_as_ushort(d)) << 16);
  *reinterpret_cast<uint2*>(out + (static_cast<int64_t>(t) * Hq + h) * kDv + tid * 4) = packed;
  if (lse && tid == 0) lse[static_cast<int64_t>(t) * Hq + h] = den > 0.f ? (m + log2f(den)) * 0.69314718055994531f : kNegInf;
}

}  // namespace

int sparse_mla_chunks(int k) { return (k + kSlots - 1) / kSlots; }

cudaError_t launch_sparse_mla(const uint16_t* q, const uint16_t* kv, int64_t nseq, int64_t kv_seq_stride, int64_t L,
                              const int32_t* seq_of, int T, int Hq, const int32_t* idx, int k, int64_t idx_stride,
                              float scale, uint16_t* out, float* lse, float* part_o, float* part_ml, uint32_t* err,
                              cudaStream_t stream) {
  MlaParams p = {};
  p.kv = kv;
  p.kv_seq_stride = kv_seq_stride;
  p.nseq = nseq;
  p.L = L;
  p.seq_of = seq_of;
  p.T = T;
  p.Hq = Hq;
  p.idx = idx;
  p.idx_stride = idx_stride;
  p.k = k;
  p.nch = sparse_mla_chunks(k);
  p.scale_log2 = scale * 1.4426950408889634f;
  p.part_o = part_o;
  p.part_ml = part_ml;
  p.err = err;
  // query rows, bf16, 128-byte swizzled K-major blocks of 64 x 128 heads
  CUtensorMap qmap;
  if (!encode_2d_map(&qmap, true, q, kDqk, static_cast<uint64_t>(T) * Hq, kDqk * 2, 64, kHM, true))
    return cudaErrorInvalidValue;
  cudaError_t e = ensure_dynamic_smem(reinterpret_cast<const void*>(sparse_mla_kernel), kSmemBytes);
  if (e != cudaSuccess) return e;
  const int64_t grid = static_cast<int64_t>(T) * p.nch;
  e = launch_pdl(sparse_mla_kernel, dim3(static_cast<unsigned>(grid)), dim3(kThreads), kSmemBytes, stream, 0, qmap, p);
  if (e != cudaSuccess) return e;
  return launch_pdl(sparse_mla_combine_kernel, dim3(static_cast<unsigned>(static_cast<int64_t>(T) * Hq)), dim3(128), 0,
                    stream, 0, static_cast<const float*>(part_o), static_cast<const float*>(part_ml), T, Hq, p.nch,
                    out, lse);
}

}  // namespace misa
