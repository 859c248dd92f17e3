// C ABI of libmisa: host-side argument checks, workspace sizing, TMA tensor
// maps and kernel launches.  See include/misa.h for the contract of each call.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstring>

#include "../../include/misa.h"
#include "launch.h"

namespace {

constexpr size_t kErrBytes = 256;

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline int64_t round_up4(int64_t x) { return (x + 3) / 4 * 4; }

inline misa_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MISA_OK : MISA_ERR_CUDA; }

uint32_t* err_word(void* ws) { return reinterpret_cast<uint32_t*>(ws); }

// 2-D map over all key rows: dim0 = 128 bf16 (256 B), dim1 = rows; box = 64 x kTmaBoxRows
// with 128-byte swizzle, the layout the UMMA descriptors expect.
misa_status make_key_map(const uint16_t* keys, int64_t rows, CUtensorMap* map) {
  return misa::encode_2d_map(map, true, keys, MISA_HEAD_DIM, static_cast<uint64_t>(rows), MISA_HEAD_DIM * 2, 64,
                             static_cast<uint32_t>(misa::kTmaBoxRows), true)
             ? MISA_OK
             : MISA_ERR_CUDA;
}

misa_status check_ws(const void* ws, size_t have, size_t need) {
  if (!ws || have < need) return MISA_ERR_WORKSPACE;
  if (!aligned16(ws)) return MISA_ERR_INVALID_ARG;
  return MISA_OK;
}

// Shared argument checks of the scoring call.
misa_status check_score_args(const uint16_t* q, const float* w, const uint16_t* keys, int64_t nkeyseq,
                             int64_t key_seq_stride, const int32_t* seq_of, const int32_t* prefix_len, int T, int H,
                             int64_t L, const int32_t* heads, int h, int q_block, const int32_t* cand, int n_cand,
                             const float* scores, int64_t row_stride) {
  if (!q || !w || !keys || !seq_of || !prefix_len || !scores) return MISA_ERR_INVALID_ARG;
  if (T < 1 || H < 1 || L < 1 || nkeyseq < 1) return MISA_ERR_INVALID_ARG;
  if (H > MISA_MAX_HEADS) return MISA_ERR_UNSUPPORTED;
  if (heads) {
    if (h < 1 || h > H || q_block < 1) return MISA_ERR_INVALID_ARG;
  }
  if (!aligned16(q) || !aligned16(keys)) return MISA_ERR_INVALID_ARG;
  if (key_seq_stride < 0 || key_seq_stride % MISA_HEAD_DIM != 0) return MISA_ERR_INVALID_ARG;
  if (key_seq_stride != 0 && key_seq_stride < L * MISA_HEAD_DIM) return MISA_ERR_INVALID_ARG;
  if (cand) {
    if (n_cand < 1 || row_stride < n_cand) return MISA_ERR_INVALID_ARG;
  } else {
    if (row_stride < L) return MISA_ERR_INVALID_ARG;
  }
  const int64_t rows = (nkeyseq - 1) * (key_seq_stride / MISA_HEAD_DIM) + L;
  if (rows + 128 >= (static_cast<int64_t>(1) << 31)) return MISA_ERR_UNSUPPORTED;  // TMA coordinates are int32
  if (L >= (static_cast<int64_t>(1) << 31) - 128) return MISA_ERR_UNSUPPORTED;
  return MISA_OK;
}

misa_status check_topk_args(const float* scores, int T, int64_t n, int64_t row_stride, const int32_t* id_map,
                            int64_t id_map_stride, int k, const int32_t* idx) {
  if (!scores || !idx) return MISA_ERR_INVALID_ARG;
  if (T < 1 || n < 1 || k < 1) return MISA_ERR_INVALID_ARG;
  if (k > MISA_MAX_TOPK || T > MISA_MAX_TOPK_ROWS) return MISA_ERR_UNSUPPORTED;
  if (n >= (static_cast<int64_t>(1) << 31)) return MISA_ERR_UNSUPPORTED;
  if (row_stride < n || row_stride % 4 != 0 || !aligned16(scores)) return MISA_ERR_INVALID_ARG;
  if (id_map && id_map_stride < n) return MISA_ERR_INVALID_ARG;
  return MISA_OK;
}

// The bf16 split of the block means: both pointers or neither, 16-byte aligned.
bool split_ok(const uint16_t* hi, const uint16_t* lo) {
  if (!hi && !lo) return true;
  return hi && lo && aligned16(hi) && aligned16(lo);
}

misa_status check_block_args(const uint16_t* q, const float* w, const float* means, const uint16_t* means_hi,
                             const uint16_t* means_lo, int64_t nseq, int64_t means_seq_stride, const int32_t* seq_of,
                             const int32_t* prefix_len, int T, int H, int64_t L, int B, int S) {
  if (!q || !w || !seq_of || !prefix_len || !split_ok(means_hi, means_lo)) return MISA_ERR_INVALID_ARG;
  if (!means && !means_hi) return MISA_ERR_INVALID_ARG;
  if (T < 1 || H < 1 || L < 1 || B < 1 || nseq < 1 || S < 1 || S > B) return MISA_ERR_INVALID_ARG;
  if (H > MISA_MAX_HEADS) return MISA_ERR_UNSUPPORTED;
  if (!aligned16(q) || (means && !aligned16(means)) || means_seq_stride < 0 || means_seq_stride % 4 != 0)
    return MISA_ERR_INVALID_ARG;
  const int64_t M = misa::num_windows(L, B, S);
  if (nseq > 1 && means_seq_stride < M * MISA_HEAD_DIM) return MISA_ERR_INVALID_ARG;
  if (M >= (static_cast<int64_t>(1) << 24) || nseq >= (static_cast<int64_t>(1) << 31)) return MISA_ERR_UNSUPPORTED;
  return MISA_OK;
}

}  // namespace

extern "C" {

const char* misa_status_string(int status) {
  switch (status) {
    case MISA_OK: return "ok";
    case MISA_ERR_INVALID_ARG: return "invalid argument";
    case MISA_ERR_UNSUPPORTED: return "unsupported size or mode";
    case MISA_ERR_WORKSPACE: return "workspace missing or too small";
    case MISA_ERR_CUDA: return "CUDA runtime error";
    case MISA_ERR_DEVICE: return "device recorded an error";
    default: return "unknown status";
  }
}

int misa_abi_version(void) { return MISA_ABI_VERSION; }

size_t misa_workspace_bytes(int op, int T, int H, int64_t L, int B, int k, int kp) {
  if (T < 0 || H < 0 || L < 0 || B < 0 || kp < 0) return 0;
  switch (op) {
    case MISA_OP_ROUTE_HEADS:
      // sized for q_block = 1 (the most routing decisions a call can have)
      if (B < 1) return 0;
      return kErrBytes + misa::router_scratch_bytes(T, H, L, B, 1);
    case MISA_OP_INDEX_SCORE:
    case MISA_OP_INDEX_DECODE:
    case MISA_OP_TOPK:
    case MISA_OP_APPEND_KEYS:
      return kErrBytes;
    case MISA_OP_HIER_RERANK:
      return kErrBytes + static_cast<size_t>(T) * round_up4(kp) * sizeof(float);
    case MISA_OP_SPARSE_MLA:
      if (k < 1) return 0;
      return kErrBytes + static_cast<size_t>(T) * misa::sparse_mla_chunks(k) * H * (MISA_MLA_DV + 2) * sizeof(float);
    case MISA_OP_HISA_BLOCK_FILTER: {
      if (B < 1) return 0;
      const int64_t M = ceil_div(L, B);
      return kErrBytes + static_cast<size_t>(T) * round_up4(M) * sizeof(float);
    }
    default:
      return 0;
  }
}

misa_status misa_error_reset(void* workspace, misa_stream_t stream) {
  if (!workspace) return MISA_ERR_INVALID_ARG;
  return cuda_status(cudaMemsetAsync(workspace, 0, sizeof(uint32_t), reinterpret_cast<cudaStream_t>(stream)));
}

misa_status misa_error_query(const void* workspace, misa_stream_t stream, uint32_t* host_bits) {
  if (!workspace || !host_bits) return MISA_ERR_INVALID_ARG;
  uint32_t v = 0;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(&v, workspace, sizeof(v), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return MISA_ERR_CUDA;
  *host_bits = v;
  return v == 0 ? MISA_OK : MISA_ERR_DEVICE;
}

int64_t misa_num_windows(int64_t L, int B, int S) {
  if (L < 1 || B < 1 || S < 1 || S > B) return 0;
  return misa::num_windows(L, B, S);
}

misa_status misa_block_stats_ex(const uint16_t* keys, int64_t nseq, int64_t L, int64_t key_seq_stride, int B, int S,
                                int pool, float* means, uint16_t* means_hi, uint16_t* means_lo,
                                misa_stream_t stream) {
  if (!keys || !means || nseq < 1 || L < 1 || B < 1 || !split_ok(means_hi, means_lo)) return MISA_ERR_INVALID_ARG;
  if (S < 1 || S > B || (pool != MISA_POOL_MEAN && pool != MISA_POOL_MAX)) return MISA_ERR_INVALID_ARG;
  if (B > 4096) return MISA_ERR_UNSUPPORTED;
  if (!aligned16(keys) || !aligned16(means) || key_seq_stride < 0 || key_seq_stride % 8 != 0)
    return MISA_ERR_INVALID_ARG;
  if (nseq > 1 && key_seq_stride < L * MISA_HEAD_DIM) return MISA_ERR_INVALID_ARG;
  return cuda_status(misa::launch_block_stats(keys, nseq, L, key_seq_stride, B, S, pool == MISA_POOL_MAX, means,
                                              means_hi, means_lo, reinterpret_cast<cudaStream_t>(stream)));
}

misa_status misa_block_stats(const uint16_t* keys, int64_t nseq, int64_t L, int64_t key_seq_stride, int B,
                             float* means, uint16_t* means_hi, uint16_t* means_lo, misa_stream_t stream) {
  return misa_block_stats_ex(keys, nseq, L, key_seq_stride, B, B, MISA_POOL_MEAN, means, means_hi, means_lo, stream);
}

misa_status misa_append_keys_ex(uint16_t* keys, int64_t nseq, int64_t key_seq_stride, int64_t L_cap,
                                const int32_t* len, const uint16_t* new_keys, int n_new, int B, int S, int pool,
                                float* means, uint16_t* means_hi, uint16_t* means_lo, int64_t means_seq_stride,
                                void* workspace, size_t workspace_bytes, misa_stream_t stream) {
  if (!keys || !len || !new_keys || !means || nseq < 1 || L_cap < 1 || n_new < 1 || B < 1 ||
      !split_ok(means_hi, means_lo))
    return MISA_ERR_INVALID_ARG;
  if (S < 1 || S > B || (pool != MISA_POOL_MEAN && pool != MISA_POOL_MAX)) return MISA_ERR_INVALID_ARG;
  if (B > 4096) return MISA_ERR_UNSUPPORTED;
  if (!aligned16(keys) || !aligned16(new_keys) || !aligned16(means) || key_seq_stride < 0 || key_seq_stride % 8 != 0)
    return MISA_ERR_INVALID_ARG;
  if (nseq > 1 && key_seq_stride < L_cap * MISA_HEAD_DIM) return MISA_ERR_INVALID_ARG;
  const int64_t M_cap = misa::num_windows(L_cap, B, S);
  if (means_seq_stride % MISA_HEAD_DIM != 0 || (nseq > 1 && means_seq_stride < M_cap * MISA_HEAD_DIM))
    return MISA_ERR_INVALID_ARG;
  misa_status st = check_ws(workspace, workspace_bytes, kErrBytes);
  if (st != MISA_OK) return st;
  return cuda_status(misa::launch_append_keys(keys, nseq, key_seq_stride, L_cap, len, new_keys, n_new, B, S,
                                              pool == MISA_POOL_MAX, means, means_hi, means_lo, means_seq_stride,
                                              err_word(workspace), reinterpret_cast<cudaStream_t>(stream)));
}

misa_status misa_append_keys(uint16_t* keys, int64_t nseq, int64_t key_seq_stride, int64_t L_cap, const int32_t* len,
                             const uint16_t* new_keys, int n_new, int B, float* means, uint16_t* means_hi,
                             uint16_t* means_lo, int64_t means_seq_stride, void* workspace, size_t workspace_bytes,
                             misa_stream_t stream) {
  return misa_append_keys_ex(keys, nseq, key_seq_stride, L_cap, len, new_keys, n_new, B, B, MISA_POOL_MEAN, means,
                             means_hi, means_lo, means_seq_stride, workspace, workspace_bytes, stream);
}

misa_status misa_route_heads_ex(const uint16_t* q, const float* w, const float* means, const uint16_t* means_hi,
                                const uint16_t* means_lo, int64_t nseq, int64_t means_seq_stride,
                                const int32_t* seq_of, const int32_t* prefix_len, int T, int H, int64_t L, int B,
                                int S, int q_block, int h, int32_t* heads, float* importance, void* workspace,
                                size_t workspace_bytes, misa_stream_t stream) {
  misa_status st =
      check_block_args(q, w, means, means_hi, means_lo, nseq, means_seq_stride, seq_of, prefix_len, T, H, L, B, S);
  if (st != MISA_OK) return st;
  if (!heads || q_block < 1 || h < 1 || h > H) return MISA_ERR_INVALID_ARG;
  if (means_seq_stride % MISA_HEAD_DIM != 0) return MISA_ERR_INVALID_ARG;  // rows of 128 means for the TMA map
  const int64_t M = misa::num_windows(L, B, S);
  st = check_ws(workspace, workspace_bytes, kErrBytes + misa::router_scratch_bytes_m(T, H, M, 1));
  if (st != MISA_OK) return st;
  // The per-decision counters of the persistent path are cleared on the stream
  // before the kernel (one small memset), so the workspace needs no
  // initialisation and a call after a wait that gave up starts clean.
  uint8_t* scratch = static_cast<uint8_t*>(workspace) + kErrBytes;
  float* partial = reinterpret_cast<float*>(scratch);
  unsigned* counters = reinterpret_cast<unsigned*>(scratch + misa::router_counters_offset_m(T, H, M));
  const int qpm = misa::route_tc_queries_per_group(H, q_block, nseq == 1 || means_seq_stride == 0);
  return cuda_status(misa::launch_route_heads_tc(q, w, means, means_hi, means_lo, means_seq_stride,
                                                 static_cast<int>(nseq), seq_of, prefix_len, T, H, L, B, S, q_block, h,
                                                 qpm, heads, importance, partial, counters, true,
                                                 err_word(workspace), reinterpret_cast<cudaStream_t>(stream)));
}

misa_status misa_route_heads(const uint16_t* q, const float* w, const float* means, const uint16_t* means_hi,
                             const uint16_t* means_lo, int64_t nseq, int64_t means_seq_stride, const int32_t* seq_of,
                             const int32_t* prefix_len, int T, int H, int64_t L, int B, int q_block, int h,
                             int32_t* heads, float* importance, void* workspace, size_t workspace_bytes,
                             misa_stream_t stream) {
  return misa_route_heads_ex(q, w, means, means_hi, means_lo, nseq, means_seq_stride, seq_of, prefix_len, T, H, L, B,
                             B, q_block, h, heads, importance, workspace, workspace_bytes, stream);
}

misa_status misa_index_score(const uint16_t* q, const float* w, const uint16_t* keys, int64_t nkeyseq,
                             int64_t key_seq_stride, const int32_t* seq_of, const int32_t* prefix_len, int T, int H,
                             int64_t L, const int32_t* heads, int h, int q_block, const int32_t* cand, int n_cand,
                             float* scores, int64_t scores_row_stride, void* workspace, size_t workspace_bytes,
                             misa_stream_t stream) {
  misa_status st = check_score_args(q, w, keys, nkeyseq, key_seq_stride, seq_of, prefix_len, T, H, L, heads, h,
                                    q_block, cand, n_cand, scores, scores_row_stride);
  if (st != MISA_OK) return st;
  st = check_ws(workspace, workspace_bytes, kErrBytes);
  if (st != MISA_OK) return st;
  CUtensorMap map;
  const CUtensorMap* mp = nullptr;
  if (!cand) {
    const int64_t rows = (nkeyseq - 1) * (key_seq_stride / MISA_HEAD_DIM) + L;
    st = make_key_map(keys, rows, &map);
    if (st != MISA_OK) return st;
    mp = &map;
  }
  misa::ScoreArgs a;
  a.q = q;
  a.w = w;
  a.keys = keys;
  a.nkeyseq = nkeyseq;
  a.key_seq_stride = key_seq_stride;
  a.seq_of = seq_of;
  a.prefix_len = prefix_len;
  a.T = T;
  a.H = H;
  a.L = L;
  a.heads = heads;
  a.h = heads ? h : H;
  a.q_block = heads ? q_block : 1;
  a.cand = cand;
  a.n_cand = cand ? n_cand : 0;
  a.scores = scores;
  a.row_stride = scores_row_stride;
  a.err = err_word(workspace);
  return cuda_status(misa::launch_index_score(mp, a, reinterpret_cast<cudaStream_t>(stream)));
}

misa_status misa_index_score_blocks(const uint16_t* q, const float* w, const uint16_t* keys, int64_t nkeyseq,
                                    int64_t key_seq_stride, const int32_t* seq_of, const int32_t* prefix_len, int T,
                                    int H, int64_t L, const int32_t* blocks, int m, int B, float* scores,
                                    int64_t scores_row_stride, void* workspace, size_t workspace_bytes,
                                    misa_stream_t stream) {
  if (!blocks || m < 1 || (B != 64 && B != 128)) return MISA_ERR_INVALID_ARG;
  const int64_t n = static_cast<int64_t>(m) * B;
  if (n >= (static_cast<int64_t>(1) << 31)) return MISA_ERR_UNSUPPORTED;
  // (the block list stands in for a candidate list of m B entries)
  misa_status st = check_score_args(q, w, keys, nkeyseq, key_seq_stride, seq_of, prefix_len, T, H, L, nullptr, H, 1,
                                    blocks, static_cast<int>(n), scores, scores_row_stride);
  if (st != MISA_OK) return st;
  st = check_ws(workspace, workspace_bytes, kErrBytes);
  if (st != MISA_OK) return st;
  CUtensorMap map;
  const int64_t rows = (nkeyseq - 1) * (key_seq_stride / MISA_HEAD_DIM) + L;
  st = make_key_map(keys, rows, &map);
  if (st != MISA_OK) return st;
  misa::ScoreArgs a;
  a.q = q;
  a.w = w;
  a.keys = keys;
  a.nkeyseq = nkeyseq;
  a.key_seq_stride = key_seq_stride;
  a.seq_of = seq_of;
  a.prefix_len = prefix_len;
  a.T = T;
  a.H = H;
  a.L = L;
  a.heads = nullptr;
  a.h = H;
  a.q_block = 1;
  a.cand = nullptr;
  a.n_cand = static_cast<int>(n);
  a.blocks = blocks;
  a.run = B;
  a.scores = scores;
  a.row_stride = scores_row_stride;
  a.err = err_word(workspace);
  return cuda_status(misa::launch_index_score(&map, a, reinterpret_cast<cudaStream_t>(stream)));
}

misa_status misa_topk(const float* scores, int T, int64_t n, int64_t row_stride, const int32_t* row_valid,
                      const int32_t* id_map, int64_t id_map_stride, int k, int32_t* idx, void* workspace,
                      size_t workspace_bytes, misa_stream_t stream) {
  misa_status st = check_topk_args(scores, T, n, row_stride, id_map, id_map_stride, k, idx);
  if (st != MISA_OK) return st;
  st = check_ws(workspace, workspace_bytes, kErrBytes);
  if (st != MISA_OK) return st;
  return cuda_status(misa::launch_topk(scores, T, n, row_stride, row_valid, id_map, id_map_stride, k, idx,
                                       reinterpret_cast<cudaStream_t>(stream)));
}

misa_status misa_index_decode(const uint16_t* q, const float* w, const uint16_t* keys, int64_t nkeyseq,
                              int64_t key_seq_stride, const uint16_t* means_hi, const uint16_t* means_lo,
                              int64_t nmeanseq, int64_t means_seq_stride, const int32_t* seq_of,
                              const int32_t* prefix_len, int T, int H, int64_t L, int B, int h, int k, int32_t* heads,
                              float* importance, float* scores, int64_t scores_row_stride, int32_t* idx,
                              void* workspace, size_t workspace_bytes, misa_stream_t stream) {
  if (!q || !w || !keys || !means_hi || !means_lo || !seq_of || !prefix_len || !heads || !scores)
    return MISA_ERR_INVALID_ARG;
  if (T < 1 || H < 1 || L < 1 || B < 1 || h < 1 || h > H || k < 1 || nkeyseq < 1 || nmeanseq < 1)
    return MISA_ERR_INVALID_ARG;
  if (!misa::decode_fused_supported(H, h, L) || k > MISA_MAX_TOPK || T > MISA_MAX_TOPK_ROWS) return MISA_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(keys) || !aligned16(means_hi) || !aligned16(means_lo) || !aligned16(scores))
    return MISA_ERR_INVALID_ARG;
  if (key_seq_stride < 0 || key_seq_stride % MISA_HEAD_DIM != 0 || (nkeyseq > 1 && key_seq_stride < L * MISA_HEAD_DIM))
    return MISA_ERR_INVALID_ARG;
  const int64_t M = ceil_div(L, B);
  if (means_seq_stride < 0 || means_seq_stride % MISA_HEAD_DIM != 0 ||
      (nmeanseq > 1 && means_seq_stride < M * MISA_HEAD_DIM))
    return MISA_ERR_INVALID_ARG;
  if (scores_row_stride < L || scores_row_stride % 4 != 0) return MISA_ERR_INVALID_ARG;
  const int64_t krows = (nkeyseq - 1) * (key_seq_stride / MISA_HEAD_DIM) + L;
  const int64_t mrows = (nmeanseq - 1) * (means_seq_stride / MISA_HEAD_DIM) + M;
  if (krows + 128 >= (static_cast<int64_t>(1) << 31) || mrows + 128 >= (static_cast<int64_t>(1) << 31) ||
      static_cast<int64_t>(T) * H >= (static_cast<int64_t>(1) << 31))
    return MISA_ERR_UNSUPPORTED;   // TMA coordinates are int32
  misa_status st = check_ws(workspace, workspace_bytes, misa_workspace_bytes(MISA_OP_INDEX_DECODE, T, H, L, B, k, 0));
  if (st != MISA_OK) return st;
  misa::DecodeArgs a;
  a.q = q;
  a.w = w;
  a.keys = keys;
  a.nkeyseq = nkeyseq;
  a.key_seq_stride = key_seq_stride;
  a.means_hi = means_hi;
  a.means_lo = means_lo;
  a.nmeanseq = nmeanseq;
  a.means_seq_stride = means_seq_stride;
  a.seq_of = seq_of;
  a.prefix_len = prefix_len;
  a.T = T;
  a.H = H;
  a.h = h;
  a.B = B;
  a.L = L;
  a.heads = heads;
  a.importance = importance;
  a.scores = scores;
  a.row_stride = scores_row_stride;
  a.err = err_word(workspace);
  const cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  misa_status rs = cuda_status(misa::launch_decode_fused(a, cs));
  if (rs != MISA_OK || !idx) return rs;   // idx NULL: heads, importance and scores only
  // the top-k starts while the last CTAs of the scoring kernel finish and
  // waits for their rows (programmatic dependent launch)
  return cuda_status(misa::launch_topk(scores, T, L, scores_row_stride, prefix_len, nullptr, 0, k, idx, cs));
}

misa_status misa_hier_rerank(const uint16_t* q, const float* w, const uint16_t* keys, int64_t nkeyseq,
                             int64_t key_seq_stride, const int32_t* seq_of, const int32_t* prefix_len, int T, int H,
                             int64_t L, const int32_t* cand, int kp, int k, float* cand_scores, int32_t* idx,
                             void* workspace, size_t workspace_bytes, misa_stream_t stream) {
  if (!cand || !idx || kp < 1 || k < 1 || k > kp || T < 1) return MISA_ERR_INVALID_ARG;
  if (k > MISA_MAX_TOPK || T > MISA_MAX_TOPK_ROWS) return MISA_ERR_UNSUPPORTED;
  misa_status st = check_ws(workspace, workspace_bytes, misa_workspace_bytes(MISA_OP_HIER_RERANK, T, H, L, 1, k, kp));
  if (st != MISA_OK) return st;
  const int64_t kp_pad = round_up4(kp);
  float* ws_scores = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + kErrBytes);
  st = check_score_args(q, w, keys, nkeyseq, key_seq_stride, seq_of, prefix_len, T, H, L, nullptr, H, 1, cand, kp,
                        ws_scores, kp_pad);
  if (st != MISA_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  misa::ScoreArgs a;
  a.q = q;
  a.w = w;
  a.keys = keys;
  a.nkeyseq = nkeyseq;
  a.key_seq_stride = key_seq_stride;
  a.seq_of = seq_of;
  a.prefix_len = prefix_len;
  a.T = T;
  a.H = H;
  a.L = L;
  a.heads = nullptr;
  a.h = H;
  a.q_block = 1;
  a.cand = cand;
  a.n_cand = kp;
  a.scores = ws_scores;
  a.row_stride = kp_pad;
  a.err = err_word(workspace);
  cudaError_t e = misa::launch_index_score(nullptr, a, s);
  if (e != cudaSuccess) return MISA_ERR_CUDA;
  e = misa::launch_topk(ws_scores, T, kp, kp_pad, nullptr, cand, kp, k, idx, s);
  if (e != cudaSuccess) return MISA_ERR_CUDA;
  if (cand_scores) {
    e = cudaMemcpy2DAsync(cand_scores, static_cast<size_t>(kp) * sizeof(float), ws_scores,
                          static_cast<size_t>(kp_pad) * sizeof(float), static_cast<size_t>(kp) * sizeof(float), T,
                          cudaMemcpyDeviceToDevice, s);
    if (e != cudaSuccess) return MISA_ERR_CUDA;
  }
  return MISA_OK;
}

misa_status hisa_block_filter_ex(const uint16_t* q, const float* w, const float* means, const uint16_t* means_hi,
                                 const uint16_t* means_lo, int64_t nseq, int64_t means_seq_stride,
                                 const int32_t* seq_of, const int32_t* prefix_len, int T, int H, int64_t L, int B,
                                 int S, int m, int32_t* blocks, int32_t* cand, float* block_scores, void* workspace,
                                 size_t workspace_bytes, misa_stream_t stream) {
  misa_status st =
      check_block_args(q, w, means, means_hi, means_lo, nseq, means_seq_stride, seq_of, prefix_len, T, H, L, B, S);
  if (st != MISA_OK) return st;
  if (!blocks || !cand || m < 1) return MISA_ERR_INVALID_ARG;
  if (means_seq_stride % MISA_HEAD_DIM != 0) return MISA_ERR_INVALID_ARG;  // rows of 128 means for the TMA map
  if (m > MISA_MAX_TOPK || T > MISA_MAX_TOPK_ROWS) return MISA_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(m) * B >= (static_cast<int64_t>(1) << 31)) return MISA_ERR_UNSUPPORTED;
  const int64_t M = misa::num_windows(L, B, S);
  const int64_t M_pad = round_up4(M);
  st = check_ws(workspace, workspace_bytes, kErrBytes + static_cast<size_t>(T) * M_pad * sizeof(float));
  if (st != MISA_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  float* bs = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + kErrBytes);
  cudaError_t e = misa::launch_hisa_block_scores_tc(q, w, means, means_hi, means_lo, means_seq_stride,
                                                    static_cast<int>(nseq), seq_of, prefix_len, T, H, L, B, S, bs,
                                                    M_pad, err_word(workspace), s);
  if (e != cudaSuccess) return MISA_ERR_CUDA;
  e = misa::launch_topk(bs, T, M, M_pad, nullptr, nullptr, 0, m, blocks, s);
  if (e != cudaSuccess) return MISA_ERR_CUDA;
  e = misa::launch_hisa_expand(blocks, prefix_len, T, m, B, S, L, cand, s);
  if (e != cudaSuccess) return MISA_ERR_CUDA;
  if (block_scores) {
    e = cudaMemcpy2DAsync(block_scores, static_cast<size_t>(M) * sizeof(float), bs,
                          static_cast<size_t>(M_pad) * sizeof(float), static_cast<size_t>(M) * sizeof(float), T,
                          cudaMemcpyDeviceToDevice, s);
    if (e != cudaSuccess) return MISA_ERR_CUDA;
  }
  return MISA_OK;
}

misa_status hisa_block_filter(const uint16_t* q, const float* w, const float* means, const uint16_t* means_hi,
                              const uint16_t* means_lo, int64_t nseq, int64_t means_seq_stride, const int32_t* seq_of,
                              const int32_t* prefix_len, int T, int H, int64_t L, int B, int m, int32_t* blocks,
                              int32_t* cand, float* block_scores, void* workspace, size_t workspace_bytes,
                              misa_stream_t stream) {
  return hisa_block_filter_ex(q, w, means, means_hi, means_lo, nseq, means_seq_stride, seq_of, prefix_len, T, H, L, B,
                              B, m, blocks, cand, block_scores, workspace, workspace_bytes, stream);
}

misa_status misa_sparse_mla(const uint16_t* q, const uint16_t* kv, int64_t nseq, int64_t kv_seq_stride, int64_t L,
                            const int32_t* seq_of, int T, int Hq, const int32_t* idx, int k, int64_t idx_stride,
                            float scale, uint16_t* out, float* lse, void* workspace, size_t workspace_bytes,
                            misa_stream_t stream) {
  if (!q || !kv || !seq_of || !idx || !out) return MISA_ERR_INVALID_ARG;
  if (T < 1 || Hq < 1 || k < 1 || L < 1 || nseq < 1 || idx_stride < k) return MISA_ERR_INVALID_ARG;
  if (Hq > 128 || k > MISA_MAX_TOPK) return MISA_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(kv) || !aligned16(out) || kv_seq_stride < 0 || kv_seq_stride % 8 != 0)
    return MISA_ERR_INVALID_ARG;
  if (nseq > 1 && kv_seq_stride < L * MISA_MLA_DQK) return MISA_ERR_INVALID_ARG;
  // query rows and grid sizes are 32-bit
  if (static_cast<int64_t>(T) * Hq >= (static_cast<int64_t>(1) << 31) ||
      static_cast<int64_t>(T) * misa::sparse_mla_chunks(k) >= (static_cast<int64_t>(1) << 31) ||
      L >= (static_cast<int64_t>(1) << 31))
    return MISA_ERR_UNSUPPORTED;
  misa_status st = check_ws(workspace, workspace_bytes, misa_workspace_bytes(MISA_OP_SPARSE_MLA, T, Hq, 0, 0, k, 0));
  if (st != MISA_OK) return st;
  const int nch = misa::sparse_mla_chunks(k);
  float* part_o = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + kErrBytes);
  float* part_ml = part_o + static_cast<size_t>(T) * nch * Hq * MISA_MLA_DV;
  return cuda_status(misa::launch_sparse_mla(q, kv, nseq, kv_seq_stride, L, seq_of, T, Hq, idx, k, idx_stride, scale,
                                             out, lse, part_o, part_ml, err_word(workspace),
                                             reinterpret_cast<cudaStream_t>(stream)));
}

misa_status misa_shard_prefix(const int32_t* prefix_len, int T, int64_t s0, int64_t L_shard, int32_t* out,
                              misa_stream_t stream) {
  if (!prefix_len || !out || T < 1 || s0 < 0 || L_shard < 1) return MISA_ERR_INVALID_ARG;
  if (L_shard >= (static_cast<int64_t>(1) << 31)) return MISA_ERR_UNSUPPORTED;
  return cuda_status(misa::launch_shard_prefix(prefix_len, T, s0, L_shard, out, reinterpret_cast<cudaStream_t>(stream)));
}

misa_status misa_gather_candidates(const float* scores, int T, int64_t n, int64_t row_stride, const int32_t* idx,
                                   int k, int64_t id_offset, float* out_scores, int32_t* out_ids,
                                   misa_stream_t stream) {
  if (!scores || !idx || !out_scores || !out_ids || T < 1 || k < 1 || n < 1 || row_stride < n || id_offset < 0)
    return MISA_ERR_INVALID_ARG;
  if (id_offset + n >= (static_cast<int64_t>(1) << 31)) return MISA_ERR_UNSUPPORTED;
  return cuda_status(misa::launch_gather_candidates(scores, T, n, row_stride, idx, k, id_offset, out_scores, out_ids,
                                                    reinterpret_cast<cudaStream_t>(stream)));
}

misa_status misa_selftest_wait_timeout(void* workspace, size_t workspace_bytes, misa_stream_t stream) {
  misa_status st = check_ws(workspace, workspace_bytes, kErrBytes);
  if (st != MISA_OK) return st;
  uint32_t* err = err_word(workspace);
  return cuda_status(misa::launch_wait_timeout_selftest(err, err + 1, reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"
