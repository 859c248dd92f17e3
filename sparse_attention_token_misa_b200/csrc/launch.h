// Internal launch interface between the C ABI (api.cu) and the kernels.
// Arguments here are already validated; every launcher is asynchronous.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace misa {

// SM count of the current device (cached; 0 on error).
int device_sm_count();
// Raise `func`'s dynamic shared-memory limit to at least `bytes` on the current
// device; cudaFuncSetAttribute runs only the first time a size is needed.
cudaError_t ensure_dynamic_smem(const void* func, int bytes);
// Resident CTAs per SM of `func` at this block size and dynamic shared memory
// (cached; 1 if the query fails).
int occupancy_blocks(const void* func, int threads, size_t smem);

cudaError_t launch_block_stats(const uint16_t* keys, int64_t nseq, int64_t L, int64_t key_seq_stride, int B,
                               float* means, cudaStream_t stream);

int router_chunks(int M);

cudaError_t launch_route_heads(const uint16_t* q, const float* w, const float* means, int64_t means_seq_stride,
                               const int32_t* seq_of, const int32_t* prefix_len, int T, int H, int64_t L, int B,
                               int q_block, int h, int nseq_means, int32_t* heads, float* importance, float* partial,
                               unsigned* counters, uint32_t* err, cudaStream_t stream);

// Tensor-core router (route_tc.cu).  qpm = queries per MMA row group (>1 only
// when the queries share one sequence's block means).
int route_tc_queries_per_group(int H, int q_block, bool shared_sequence);
cudaError_t launch_route_heads_tc(const uint16_t* q, const float* w, const float* means, int64_t means_seq_stride,
                                  int nseq, const int32_t* seq_of, const int32_t* prefix_len, int T, int H, int64_t L,
                                  int B, int q_block, int h, int qpm, int32_t* heads, float* importance,
                                  float* partial, unsigned* counters, uint32_t* err, cudaStream_t stream);

// Bytes of router scratch: partial importances [T][ceil(M/32)][H] fp32 followed
// (at a 256-byte boundary) by one counter per routing decision.
size_t router_scratch_bytes(int T, int H, int64_t L, int B, int q_block);
size_t router_counters_offset(int T, int H, int64_t L, int B);

cudaError_t launch_hisa_block_scores(const uint16_t* q, const float* w, const float* means, int64_t means_seq_stride,
                                     const int32_t* seq_of, const int32_t* prefix_len, int T, int H, int64_t L, int B,
                                     int nseq_means, float* bscore, int64_t bs_stride, uint32_t* err,
                                     cudaStream_t stream);

cudaError_t launch_hisa_expand(const int32_t* blocks, const int32_t* prefix_len, int T, int m, int B, int64_t L,
                               int32_t* cand, cudaStream_t stream);

// Rows per TMA box of the key map (a 128-key tile is loaded as 128 / kTmaBoxRows
// boxes per 64-element K half; the host encodes the map with this box height).
#ifndef MISA_TMA_BOX_ROWS
#define MISA_TMA_BOX_ROWS 64
#endif
constexpr int kTmaBoxRows = MISA_TMA_BOX_ROWS;

struct ScoreArgs {
  const uint16_t* q;
  const float* w;
  const uint16_t* keys;
  int64_t nkeyseq;
  int64_t key_seq_stride;
  const int32_t* seq_of;
  const int32_t* prefix_len;
  int T;
  int H;
  int64_t L;
  const int32_t* heads;
  int h;
  int q_block;
  const int32_t* cand;
  int n_cand;
  float* scores;
  int64_t row_stride;
  uint32_t* err;
};

// MMA column count per query for a head count (power of two; >= 16 unless the
// queries of a group share one key cache).
int score_mode_hp(int h_eff, bool shared_groups);

cudaError_t launch_index_score(const CUtensorMap* tmap, const ScoreArgs& a, cudaStream_t stream);

size_t topk_smem_bytes();

cudaError_t launch_topk(const float* scores, int T, int64_t n, int64_t row_stride, const int32_t* row_valid,
                        const int32_t* id_map, int64_t id_map_stride, int k, int32_t* idx, cudaStream_t stream);

}  // namespace misa
