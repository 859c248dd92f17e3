// misa_route_heads_noalloc: the head router for callers that cannot hand the
// library a workspace.
//
// Some hosts cannot allocate device memory at the point where they call the
// router: an inference engine that has reserved all device memory up front and
// exposes no allocator to its plug-ins, or a latency-critical serving loop in
// which cudaMalloc / cudaFree are off limits because they may synchronise the
// whole device.  This entry point takes the same inputs and outputs as
// misa_route_heads but keeps the router's per-chunk partial importances in a
// fixed array compiled into the library instead of a caller workspace.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/misa.h"
#include "launch.h"

namespace {

// Scratch for the partial head importances, [T][ceil(M/32)][H] fp32, and one
// counter per routing decision.  Every device that loads the library holds
// these bytes until the process exits.
constexpr size_t kScratchBytes = MISA_ROUTE_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_route_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_route_scratch on the current device.  In host code the
// array's name only stands in for the symbol; the address the kernel may use
// comes from cudaGetSymbolAddress, looked up once per device with that device
// current.
misa_status scratch_on_current_device(float** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MISA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return MISA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_route_scratch) != cudaSuccess || !p) return MISA_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = static_cast<float*>(g_scratch_addr[dev]);
  return MISA_OK;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" {

misa_status misa_route_heads_noalloc(const uint16_t* q, const float* w, const float* means, int64_t nseq,
                                     int64_t means_seq_stride, const int32_t* seq_of, const int32_t* prefix_len,
                                     int T, int H, int64_t L, int B, int q_block, int h, int32_t* heads,
                                     float* importance, misa_stream_t stream) {
  // Same argument rules as misa_route_heads.
  if (!q || !w || !means || !seq_of || !prefix_len || !heads) return MISA_ERR_INVALID_ARG;
  if (T < 1 || H < 1 || L < 1 || B < 1 || nseq < 1 || q_block < 1 || h < 1 || h > H) return MISA_ERR_INVALID_ARG;
  if (H > MISA_MAX_HEADS) return MISA_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(means) || means_seq_stride < 0 || means_seq_stride % MISA_HEAD_DIM != 0)
    return MISA_ERR_INVALID_ARG;
  const int64_t M = (L + B - 1) / B;
  if (nseq > 1 && means_seq_stride < M * MISA_HEAD_DIM) return MISA_ERR_INVALID_ARG;
  if (M >= (static_cast<int64_t>(1) << 24) || nseq >= (static_cast<int64_t>(1) << 31)) return MISA_ERR_UNSUPPORTED;
  // The partial importances and the per-decision counters must fit in the
  // fixed scratch array.
  if (misa::router_scratch_bytes(T, H, L, B, q_block) > kScratchBytes) return MISA_ERR_UNSUPPORTED;

  float* partial = nullptr;
  misa_status st = scratch_on_current_device(&partial);
  if (st != MISA_OK) return st;
  unsigned* counters = reinterpret_cast<unsigned*>(reinterpret_cast<uint8_t*>(partial) +
                                                   misa::router_counters_offset(T, H, L, B));
  // The launcher clears the counters (the only part that must start at zero)
  // on the stream before the kernel; the partials are written before they are
  // read.  Device-side index checks clamp a bad seq_of without reporting it
  // (there is no error word).
  const int qpm = misa::route_tc_queries_per_group(H, q_block, nseq == 1 || means_seq_stride == 0);
  cudaError_t e = misa::launch_route_heads_tc(q, w, means, nullptr, nullptr, means_seq_stride, static_cast<int>(nseq), seq_of,
                                              prefix_len, T, H, L, B, B, q_block, h, qpm, heads, importance, partial,
                                              counters, true, nullptr, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MISA_OK : MISA_ERR_CUDA;
}

}  // extern "C"
