// Internal launch interface between the C ABI (api.cu) and the kernels.
// Arguments here are already validated; every launcher is asynchronous.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <utility>

namespace misa {

// SM count of the current device (cached; 0 on error).
int device_sm_count();
// Raise `func`'s dynamic shared-memory limit to at least `bytes` on the current
// device; cudaFuncSetAttribute runs only the first time a size is needed.
cudaError_t ensure_dynamic_smem(const void* func, int bytes);
// 2-D TMA map over `rows` rows of `inner` elements (bf16 or fp32), rows
// `row_bytes` apart; box = box_inner x box_rows; optional 128-byte swizzle.
bool encode_2d_map(CUtensorMap* map, bool bf16, const void* base, uint64_t inner, uint64_t rows, uint64_t row_bytes,
                   uint32_t box_inner, uint32_t box_rows, bool swizzle128);
// Resident CTAs per SM of `func` at this block size and dynamic shared memory
// (cached; 1 if the query fails).
int occupancy_blocks(const void* func, int threads, size_t smem);

// Launch with programmatic stream serialization (the kernel may start while the
// previous kernel of the stream is still running; it calls pdl_wait_inputs()
// before reading anything) and an optional cluster size.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       int cluster_x, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  int n = 0;
  attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[n].val.programmaticStreamSerializationAllowed = 1;
  ++n;
  if (cluster_x > 0) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster_x;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// Windows of B keys every S keys over a cache of L keys: 1 + ceil(max(L - B, 0) / S).
int64_t num_windows(int64_t L, int64_t B, int64_t S);
cudaError_t launch_block_stats(const uint16_t* keys, int64_t nseq, int64_t L, int64_t key_seq_stride, int B, int S,
                               bool pool_max, float* means, uint16_t* means_hi, uint16_t* means_lo,
                               cudaStream_t stream);
cudaError_t launch_append_keys(uint16_t* keys, int64_t nseq, int64_t key_seq_stride, int64_t L_cap,
                               const int32_t* len, const uint16_t* new_keys, int n_new, int B, int S, bool pool_max,
                               float* means, uint16_t* means_hi, uint16_t* means_lo, int64_t means_seq_stride,
                               uint32_t* err, cudaStream_t stream);

int router_chunks(int M);

// Tensor-core router (route_tc.cu).  qpm = queries per MMA row group (>1 only
// when the queries share one sequence's block means).
int route_tc_queries_per_group(int H, int q_block, bool shared_sequence);
// S: the window stride of the block statistics (S = B: plain blocks).
cudaError_t launch_route_heads_tc(const uint16_t* q, const float* w, const float* means, const uint16_t* means_hi,
                                  const uint16_t* means_lo, int64_t means_seq_stride,
                                  int nseq, const int32_t* seq_of, const int32_t* prefix_len, int T, int H, int64_t L,
                                  int B, int S, int q_block, int h, int qpm, int32_t* heads, float* importance,
                                  float* partial, unsigned* counters, bool clear_counters, uint32_t* err,
                                  cudaStream_t stream);

// Bytes of router scratch for M block statistics: partial importances (at most
// [T][ceil(M/32)][H] fp32) followed, at a 256-byte boundary, by one counter
// per routing decision.
size_t router_scratch_bytes_m(int T, int H, int64_t M, int q_block);
size_t router_counters_offset_m(int T, int H, int64_t M);
// The same for M = ceil(L / B) plain blocks.
size_t router_scratch_bytes(int T, int H, int64_t L, int B, int q_block);
size_t router_counters_offset(int T, int H, int64_t L, int B);

cudaError_t launch_hisa_block_scores_tc(const uint16_t* q, const float* w, const float* means,
                                        const uint16_t* means_hi, const uint16_t* means_lo, int64_t means_seq_stride,
                                        int nseq, const int32_t* seq_of, const int32_t* prefix_len, int T, int H,
                                        int64_t L, int B, int S, float* bscore,
                                        int64_t bs_stride, uint32_t* err, cudaStream_t stream);

// Bounded-wait self-test (selftest.cu): result[0] = 1 if the wait returned true.
cudaError_t launch_wait_timeout_selftest(uint32_t* err, uint32_t* result, cudaStream_t stream);

// Key-sharded indexer helpers (shard.cu).
cudaError_t launch_shard_prefix(const int32_t* prefix_len, int T, int64_t s0, int64_t L_shard, int32_t* out,
                                cudaStream_t stream);
cudaError_t launch_gather_candidates(const float* scores, int T, int64_t n, int64_t row_stride, const int32_t* idx,
                                     int k, int64_t id_offset, float* out_scores, int32_t* out_ids,
                                     cudaStream_t stream);

// Sparse attention over selected tokens (sparse_mla.cu): chunks of 256 index
// slots per query, partial results in part_o [T][nch][Hq][512] and part_ml
// [T][nch][Hq][2], merged by a second kernel into out / lse.
int sparse_mla_chunks(int k);
cudaError_t launch_sparse_mla(const uint16_t* q, const uint16_t* kv, int64_t nseq, int64_t kv_seq_stride, int64_t L,
                              const int32_t* seq_of, int T, int Hq, const int32_t* idx, int k, int64_t idx_stride,
                              float scale, uint16_t* out, float* lse, float* part_o, float* part_ml, uint32_t* err,
                              cudaStream_t stream);

cudaError_t launch_hisa_expand(const int32_t* blocks, const int32_t* prefix_len, int T, int m, int B, int S,
                               int64_t L, int32_t* cand, cudaStream_t stream);

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
  const int32_t* blocks = nullptr;   // block mode (cand NULL): [T][n_cand / run] key blocks
  int run = 0;
  float* scores;
  int64_t row_stride;
  uint32_t* err;
};

// MMA column count per query for a head count (power of two; >= 16 unless the
// queries of a group share one key cache).
int score_mode_hp(int h_eff, bool shared_groups);

cudaError_t launch_index_score(const CUtensorMap* tmap, const ScoreArgs& a, cudaStream_t stream);

// Router + routed scoring of a decode step in one persistent kernel
// (decode_fused.cu); the top-k of its score rows is launch_topk's.
struct DecodeArgs {
  const uint16_t* q;
  const float* w;
  const uint16_t* keys;
  int64_t nkeyseq, key_seq_stride;
  const uint16_t* means_hi;
  const uint16_t* means_lo;
  int64_t nmeanseq, means_seq_stride;
  const int32_t* seq_of;
  const int32_t* prefix_len;
  int T, H, h, B;
  int64_t L;
  int32_t* heads;
  float* importance;
  float* scores;
  int64_t row_stride;
  uint32_t* err;
};
bool decode_fused_supported(int H, int h, int64_t L);
cudaError_t launch_decode_fused(const DecodeArgs& a, cudaStream_t stream);

size_t topk_smem_bytes();

cudaError_t launch_topk(const float* scores, int T, int64_t n, int64_t row_stride, const int32_t* row_valid,
                        const int32_t* id_map, int64_t id_map_stride, int k, int32_t* idx, cudaStream_t stream);

}  // namespace misa
