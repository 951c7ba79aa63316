// Internal definitions shared by the host-side API and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/twell.h"

namespace twell {

// Bounded device waits: give up after ~2 s of wall time (a healthy wait in these
// kernels lasts microseconds) or this many polls, whichever comes first.
constexpr uint64_t kWaitTimeoutNs = 2000000000ull;
constexpr uint32_t kWaitMaxIters = 1u << 30;

// Tile shapes of the tensor-core kernels.
constexpr int kBlockM = 128;   // tokens per accumulator tile (TMEM lanes)
constexpr int kBlockK = 64;    // K elements per pipeline stage (one 128-byte swizzle row)
constexpr int kUmmaK = 16;     // K per tcgen05.mma (bf16)
constexpr int kMaxEllFused = 64;

// Device view of a TwELL matrix plus the overflow staging area in the workspace.
struct PackTarget {
  int M, f, tw, E, T;
  uint16_t *vals;
  uint8_t *idx;
  uint16_t *nnz;
  int cap;
  int32_t *n_ovf;
  int32_t *ovf_pos;
  uint16_t *ovf_dense;
  int32_t *status;
  // workspace
  int32_t *stage_ctr;      // [1] number of staged overflow segments (unsorted)
  int32_t *row_ovf;        // [M] overflow pairs per token
  int32_t *row_prefix;     // [M] exclusive prefix of row_ovf
  int32_t *stage_pos;      // [cap] r*T+t of each staged segment
  uint16_t *stage_dense;   // [cap][tw] staged dense segments
};

// Read-only device view used by the down-projection kernels.
struct TwellView {
  int M, f, tw, E, T;
  const uint16_t *vals;
  const uint8_t *idx;
  const uint16_t *nnz;
  int cap;
  const int32_t *n_ovf;
  const int32_t *ovf_pos;
  const uint16_t *ovf_dense;
  int32_t *status;
};

// Argument rules shared by the entry points (twell_api.cu).  Each returns
// TWELL_OK or the status the call reports; none touches the GPU.
bool a16(const void *p);                 // 16-byte aligned (NULL passes)
bool valid_tile(int tile_w);
twell_status check_shape(int M, int d_ff, int tile_w, int ell_w);
twell_status check_matrix(const twell_matrix *a, int M, int d_ff, int tile_w, int ell_w);
// twell_pack's rules without the workspace: shape, then (M > 0) h and the
// destination matrix.  M == 0 returns TWELL_OK before `h` and `out` are read.
twell_status check_pack_args(const uint16_t *h, int M, int d_ff, int ld_h, int tile_w, int ell_w,
                             const twell_matrix *out);

// Workspace carve-up (every region 256-byte aligned).
struct WsLayout {
  size_t ctr, row_ovf, row_prefix, stage_pos, stage_dense, total;
};

inline size_t align256(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }

inline WsLayout ws_layout(int M, int tile_w, int cap) {
  WsLayout L;
  size_t o = 0;
  L.ctr = o;         o = align256(o + 64);
  L.row_ovf = o;     o = align256(o + sizeof(int32_t) * static_cast<size_t>(M));
  L.row_prefix = o;  o = align256(o + sizeof(int32_t) * static_cast<size_t>(M));
  L.stage_pos = o;   o = align256(o + sizeof(int32_t) * static_cast<size_t>(cap));
  L.stage_dense = o; o = align256(o + 2 * static_cast<size_t>(cap) * tile_w);
  L.total = o;
  return L;
}

// Launch `kern` on stream `s` through cudaLaunchKernelEx.  With `pdl` the grid
// may be scheduled while the previous kernel on the stream is still finishing
// (programmatic dependent launch): the kernel then runs griddep_wait() before it
// touches that kernel's results.  Only launches whose predecessor is known --
// the library's own previous kernel of the same call -- set it.  `cluster` > 1
// groups CTAs along x into clusters of that size.
template <typename... KArgs, typename... Args>
cudaError_t launch_k(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                     bool pdl, unsigned cluster, Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  unsigned n = 0;
  if (cluster > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  if (pdl) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<Args &&>(args)...);
}

// ---------------------------------------------------------------------------
// Launchers (defined next to their kernels).  Each returns cudaSuccess or the
// launch error; none synchronises.
// ---------------------------------------------------------------------------
cudaError_t launch_pack_dense(const uint16_t *h, int ld_h, const PackTarget &t, cudaStream_t s);
cudaError_t launch_overflow_finalize(const PackTarget &t, cudaStream_t s);
// Per token: l1[r] = sum over tiles of l1_part[r][t] and nnz_row[r] = sum of the
// TwELL counts (either output may be NULL), in a fixed order; a dependent launch
// after the producer's backup ordering.
cudaError_t launch_stats_reduce(const PackTarget &t, const float *l1_part, float *l1, int32_t *nnz_row,
                                cudaStream_t s);

struct UpArgs {
  const uint16_t *x, *w_up, *w_gate, *b;
  int M, d, f;
  float *z_debug;
  float *l1_part;   // NULL, or [M][T] fp32: per (token, tile) sum of |h| (statistics)
};
cudaError_t launch_up_pack(const UpArgs &a, const PackTarget &t, int num_sms, cudaStream_t s);

// Split schedule of the tensor-core down-projection (128-token x 512-column
// tiles): the tiles' K steps, in hidden-tile chunks, are dealt out evenly over
// up to kMaxSplitCtas persistent CTAs, so every SM gets the same share however
// the tile count falls against the SM count.  A tile shared by several CTAs is
// summed from their fp32 partial tiles, in CTA order, by the last one to finish.
// Workspace: one arrival counter per CTA (zeroed by launch_block_path before
// every launch) and two partial tiles per CTA.
constexpr int kMaxSplitCtas = 160;
constexpr size_t kSplitPartBytes = static_cast<size_t>(kBlockM) * 512 * 4;
struct SplitWs {
  float *part;     // [2 * kMaxSplitCtas][kSplitPartBytes / 4], or NULL: no split
  int32_t *ctr;    // [kMaxSplitCtas]
};
// Workspace bytes of the split schedule for M tokens and d_model columns
// (0 when that shape never takes the split kernel).
size_t split_ws_bytes(int M, int d_model);

// blk_path: NULL (the kernel owns every token block) or one int per 128-token
// block: 0 = gather path owns it, 1 = tensor-core path owns it.
cudaError_t launch_spmm_gather(const TwellView &v, const uint16_t *w_down, int d, uint16_t *y,
                               const int32_t *blk_path, bool pdl, cudaStream_t s);
cudaError_t launch_spmm_mma(const TwellView &v, const uint16_t *w_down, int d, uint16_t *y,
                            const int32_t *blk_path, const SplitWs &split, int num_sms, bool pdl,
                            cudaStream_t s);
// Per 128-token block (256 with CTA pairs): the down path by density against
// `crossover` (a negative crossover sends every block to the tensor cores); also
// zeroes the split schedule's arrival counters (split_ctr may be NULL).
cudaError_t launch_block_path(const TwellView &v, float crossover, int32_t *blk_path, int32_t *split_ctr,
                              bool pdl, cudaStream_t s);

// Zero the status word and the staging counters before a producer; the
// producers (launch_up_pack, launch_up_pack_decode, launch_pack_dense) are
// dependent launches that must directly follow it.
cudaError_t launch_pack_reset(const PackTarget &t, cudaStream_t s);

// Exclusive scan of t.row_ovf into t.row_prefix; the total goes to *t.n_ovf
// (TWELL_ERR_OVERFLOW_CAPACITY in t.status when above t.cap).
cudaError_t launch_row_scan(const PackTarget &t, bool pdl, cudaStream_t s);

// Whole-token overflow form built from the per-(token, tile) form.
cudaError_t launch_tok_flags(const TwellView &a, int32_t *flag, cudaStream_t s);
cudaError_t launch_tok_build(const TwellView &a, const int32_t *flag, const int32_t *rank, const int32_t *n_tok,
                             int cap, uint16_t *main_nnz, int32_t *tok_pos, uint16_t *d_vals, uint8_t *d_idx,
                             uint16_t *d_nnz, cudaStream_t s);
cudaError_t launch_tok_scatter(const int32_t *n_tok, int cap, const int32_t *tok_pos, const uint16_t *y_dense,
                               int d, uint16_t *y, cudaStream_t s);

// Backward pass (non-gated): dZ = (dY W_down^T) at the forward's pattern, and
// the TwELL transpose (tiles of 128 tokens; optional per-(unit, token tile) sums).
cudaError_t launch_sddmm(const TwellView &h, const uint16_t *dy, const uint16_t *w_down, int d,
                         uint16_t *dz_vals, uint16_t *dz_ovf, int num_sms, cudaStream_t s);
cudaError_t launch_twell_transpose(const TwellView &a, const PackTarget &out, float *sum_part, bool pdl,
                                   cudaStream_t s);

// Decode-size batches (M <= 256): tokens on the MMA N side, weights streamed
// over all SMs (up: one CTA per 128 hidden units; down: split-K clusters).
bool decode_up_eligible(int M, int d_ff, int tile_w);
bool decode_down_eligible(int M);
cudaError_t launch_up_pack_decode(const UpArgs &a, const PackTarget &t, int num_sms, cudaStream_t s);
// touch_ws: dec_touch_ws_bytes(M, d_ff) bytes of workspace for the touched-unit
// bitmap (NULL: always the streaming kernel).
cudaError_t launch_spmm_decode(const TwellView &v, const uint16_t *w_down, int d, uint16_t *y,
                               uint32_t *touch_ws, int num_sms, bool pdl, cudaStream_t s);
size_t dec_touch_ws_bytes(int M, int d_ff);

// Down path of a 128-token block (the block-path array the down kernels share).
constexpr int kPathGather = 0;   // CUDA-core gather (k_spmm_gather)
constexpr int kPathDense = 1;    // tensor cores on dense h tiles rebuilt from TwELL (k_spmm_mma)
constexpr int kPathSparse = 2;   // 2:4 structured-sparse tensor cores + excess fix-up (k_spmm_sp)

// 2:4 split of h for the structured-sparse down path: per token, the nonzeros
// beyond the first two of an aligned group of 4 hidden units ("excess") are
// listed (at most kSpXc per token; a 256-token group with more takes the dense
// tensor-core path) and added on CUDA cores in the epilogue.
constexpr int kSpXc = 32;
bool sp_eligible(const TwellView &v, int d_model);
// Workspace of the 2:4 path: per-token excess counts, lists and fp32 excess
// products [M][d_model], the kept values [M][d_ff / 2] and their MMA position codes.
size_t sp_ws_bytes(int M, int d_ff, int d_model);
// k_sp_prep then k_sp_decide: the 2:4 operand, excess lists and products, and
// per 256-token group its down path (gather below gather_below; 2:4 when
// allow_sparse and no token exceeds kSpXc; else dense); also zeroes the dense
// kernel's split counters (split_ctr may be NULL).  sp_ws: the sp_ws_bytes region.
cudaError_t launch_sp_prep(const TwellView &v, const uint16_t *w_down, int d, void *sp_ws, float gather_below,
                           bool allow_sparse, int32_t *blk_path, int32_t *split_ctr, bool pdl, cudaStream_t s);
cudaError_t launch_spmm_sp(const TwellView &v, const uint16_t *w_down, int d, uint16_t *y, const int32_t *blk_path,
                           void *sp_ws, int num_sms, bool pdl, cudaStream_t s);

// Density (nonzeros / (rows * d_ff)) of a 128-token block at or above which the
// AUTO down-projection uses the tensor-core path.  Chosen from measurement.
constexpr float kDownCrossoverDensity = 0.006f;

// Driver entry point for cuTensorMapEncodeTiled (resolved at run time so the
// library loads on machines without a driver).
// A K-major bf16 matrix [rows][K] (K % 64 == 0) as a 3-D tensor (64 elements,
// rows, K / 64 chunks) with 128-byte swizzle: one box of box_rows x `chunks`
// chunks lands in shared memory as `chunks` consecutive [box_rows][64] tiles,
// the layout of as many separate 2-D boxes, in one TMA request (the TMA unit's
// throughput is bounded per request as well as per byte).
CUresult encode_tensor_map_kchunks(CUtensorMap *map, const void *base, uint64_t K, uint64_t rows,
                                   uint32_t box_rows, uint32_t chunks);

CUresult encode_tensor_map_2d(CUtensorMap *map, const void *base, uint64_t inner, uint64_t outer,
                              uint64_t row_pitch_bytes, uint32_t box_inner, uint32_t box_outer,
                              CUtensorMapSwizzle swizzle,
                              CUtensorMapDataType dtype = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16);

}  // namespace twell
