// twell_pack_noalloc: the dense-h -> TwELL packer for callers that cannot hand
// the library a workspace.
//
// twell_pack needs caller-provided scratch (the unordered overflow staging area
// and per-token counters).  Some callers have no way to obtain that memory at
// the point they pack: a serving runtime that reserved the whole device up front
// for weights and its KV-cache pool and forbids cudaMalloc on the request path,
// or a plugin host that passes only input/output buffers and owns no workspace
// to lend.  This variant keeps the scratch in a fixed, library-owned device
// array instead, so the call itself allocates nothing.
//
// The array is a file-scope __device__ variable: it exists on every GPU that
// loads this library, from module load until process exit, whether or not the
// entry point is ever called.  Host code cannot use the array's name as a
// device address; the address is looked up once per device with
// cudaGetSymbolAddress (with that device current) and passed to the kernels.
#include <mutex>

#include "twell_internal.h"

namespace twell {
namespace {

// Upper bound on the scratch one call may use.
constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;   // 4 MiB

__device__ __align__(256) uint8_t g_pack_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void *g_scratch_dev[kMaxDevices] = {nullptr};

// Device address of g_pack_scratch on the current device (looked up once).
cudaError_t scratch_address(void **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (g_scratch_dev[dev] == nullptr) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_pack_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_dev[dev] = p;
  }
  *out = g_scratch_dev[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace twell

using namespace twell;

extern "C" twell_status twell_pack_noalloc(const uint16_t *h, int M, int d_ff, int ld_h,
                                           int tile_w, int ell_w, const twell_matrix *out,
                                           void *stream) {
  // -- the same argument rules as twell_pack (shared code, so the two cannot drift)
  const twell_status st = check_pack_args(h, M, d_ff, ld_h, tile_w, ell_w, out);
  if (st != TWELL_OK || M == 0) return st;

  // -- the scratch this call needs must fit the fixed array
  const WsLayout L = ws_layout(M, tile_w, out->ovf_capacity);
  if (L.total > kNoAllocScratchBytes) return TWELL_ERR_WORKSPACE;

  void *scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess) return TWELL_ERR_CUDA;
  uint8_t *base = static_cast<uint8_t *>(scratch);

  PackTarget t;
  t.M = M; t.f = d_ff; t.tw = tile_w; t.E = ell_w; t.T = d_ff / tile_w;
  t.vals = out->vals; t.idx = out->idx; t.nnz = out->nnz;
  t.cap = out->ovf_capacity; t.n_ovf = out->n_ovf; t.ovf_pos = out->ovf_pos;
  t.ovf_dense = out->ovf_dense; t.status = out->status;
  t.stage_ctr = reinterpret_cast<int32_t *>(base + L.ctr);
  t.row_ovf = reinterpret_cast<int32_t *>(base + L.row_ovf);
  t.row_prefix = reinterpret_cast<int32_t *>(base + L.row_prefix);
  t.stage_pos = reinterpret_cast<int32_t *>(base + L.stage_pos);
  t.stage_dense = reinterpret_cast<uint16_t *>(base + L.stage_dense);

  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // The array keeps whatever the previous call left in it: the status word, the
  // staging counter and the per-token overflow counts must start at zero.
  if (launch_pack_reset(t, s) != cudaSuccess) return TWELL_ERR_CUDA;
  if (launch_pack_dense(h, ld_h, t, s) != cudaSuccess) return TWELL_ERR_CUDA;
  return launch_overflow_finalize(t, s) == cudaSuccess ? TWELL_OK : TWELL_ERR_CUDA;
}
