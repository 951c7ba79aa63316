// Host side of the C ABI declared in include/twell.h: argument validation,
// workspace carve-up, tensor-map encoding and kernel launch order.  Nothing here
// computes on the host; every step of the layer runs in the kernels.
#include <cstring>
#include <mutex>

#include "twell_internal.h"

namespace twell {

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

int sm_count() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (dev < 0 || dev >= 64) return 0;
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    cache[dev] = n;
  }
  return cache[dev];
}

// Workspace regions: overflow staging + per-block path flags.
struct Ws {
  WsLayout L;
  size_t blk_path;   // [M / 128 + 1] i32: down path of each 128-token block
  size_t l1_part;    // [M][T] fp32: per (token, tile) sums of |h| (statistics)
  size_t split;      // split schedule of the tensor-core down-projection (present
                     // when d_model is given and the shape can use it)
  size_t split_bytes;
  size_t sp;         // excess lists of the 2:4 down path (present when d_model is
                     // given and the shape can use it)
  size_t sp_bytes;
  size_t touch;      // touched-unit bitmap of the decode-size down kernel
  size_t touch_bytes;
  size_t total;
};

// d_model = 0: the regions of the calls that never run the down-projection.
Ws ws_plan(int M, int d_ff, int tile_w, int ell_w, int cap, int d_model = 0) {
  Ws w;
  w.L = ws_layout(M, tile_w, cap);
  w.blk_path = w.L.total;
  w.l1_part = align256(w.blk_path + sizeof(int32_t) * static_cast<size_t>((M + kBlockM - 1) / kBlockM + 1));
  w.split = align256(w.l1_part + sizeof(float) * static_cast<size_t>(M) * (d_ff / tile_w));
  w.split_bytes = d_model > 0 ? split_ws_bytes(M, d_model) : 0;
  w.sp = align256(w.split + w.split_bytes);
  TwellView v = {};
  v.M = M; v.f = d_ff; v.tw = tile_w; v.E = ell_w; v.T = d_ff / tile_w;
  w.sp_bytes = (d_model > 0 && sp_eligible(v, d_model)) ? sp_ws_bytes(M, d_ff, d_model) : 0;
  w.touch = align256(w.sp + w.sp_bytes);
  w.touch_bytes = d_model > 0 ? dec_touch_ws_bytes(M, d_ff) : 0;
  w.total = align256(w.touch + w.touch_bytes);
  return w;
}

SplitWs split_ptrs(const Ws &w, void *ws) {
  SplitWs sp;
  sp.part = nullptr;
  sp.ctr = nullptr;
  if (w.split_bytes > 0) {
    uint8_t *base = static_cast<uint8_t *>(ws) + w.split;
    sp.ctr = reinterpret_cast<int32_t *>(base);
    sp.part = reinterpret_cast<float *>(base + 1024);
  }
  return sp;
}

PackTarget make_target(const twell_matrix *a, void *ws) {
  const Ws w = ws_plan(a->M, a->d_ff, a->tile_w, a->ell_w, a->ovf_capacity);
  uint8_t *base = static_cast<uint8_t *>(ws);
  PackTarget t;
  t.M = a->M; t.f = a->d_ff; t.tw = a->tile_w; t.E = a->ell_w; t.T = a->d_ff / a->tile_w;
  t.vals = a->vals; t.idx = a->idx; t.nnz = a->nnz;
  t.cap = a->ovf_capacity; t.n_ovf = a->n_ovf; t.ovf_pos = a->ovf_pos; t.ovf_dense = a->ovf_dense;
  t.status = a->status;
  t.stage_ctr = reinterpret_cast<int32_t *>(base + w.L.ctr);
  t.row_ovf = reinterpret_cast<int32_t *>(base + w.L.row_ovf);
  t.row_prefix = reinterpret_cast<int32_t *>(base + w.L.row_prefix);
  t.stage_pos = reinterpret_cast<int32_t *>(base + w.L.stage_pos);
  t.stage_dense = reinterpret_cast<uint16_t *>(base + w.L.stage_dense);
  return t;
}

TwellView make_view(const twell_matrix *a) {
  TwellView v;
  v.M = a->M; v.f = a->d_ff; v.tw = a->tile_w; v.E = a->ell_w; v.T = a->d_ff / a->tile_w;
  v.vals = a->vals; v.idx = a->idx; v.nnz = a->nnz;
  v.cap = a->ovf_capacity; v.n_ovf = a->n_ovf; v.ovf_pos = a->ovf_pos; v.ovf_dense = a->ovf_dense;
  v.status = a->status;
  return v;
}

twell_status from_cuda(cudaError_t e) { return e == cudaSuccess ? TWELL_OK : TWELL_ERR_CUDA; }

// Reset the status word and the overflow staging counters before a producer
// runs (one kernel; the producer overlaps it as a dependent launch).
twell_status reset_for_pack(const PackTarget &t, cudaStream_t s) {
  return from_cuda(launch_pack_reset(t, s));
}

twell_status check_ws(void *ws, size_t ws_bytes, int M, int d_ff, int tile_w, int ell_w, int cap, int d_model = 0) {
  const Ws w = ws_plan(M, d_ff, tile_w, ell_w, cap, d_model);
  if (ws == nullptr || !a16(ws) || ws_bytes < w.total) return TWELL_ERR_WORKSPACE;
  return TWELL_OK;
}

// l1 / nnz_row: optional per-token statistics (twell_up_pack_stats).
twell_status up_pack_checked(const uint16_t *x, const uint16_t *W_up, const uint16_t *W_gate,
                             const uint16_t *b, int M, int d_model, int d_ff, int tile_w, int ell_w,
                             const twell_matrix *out, float *z_debug, void *ws, size_t ws_bytes,
                             cudaStream_t s, float *l1 = nullptr, int32_t *nnz_row = nullptr) {
  if (M == 0) return TWELL_OK;
  const PackTarget t = make_target(out, ws);
  const int sms = sm_count();
  if (sms <= 0) return TWELL_ERR_CUDA;
  twell_status st = reset_for_pack(t, s);
  if (st != TWELL_OK) return st;
  const Ws w = ws_plan(M, d_ff, tile_w, ell_w, out->ovf_capacity);
  float *l1_part = (l1 != nullptr) ? reinterpret_cast<float *>(static_cast<uint8_t *>(ws) + w.l1_part)
                                   : nullptr;
  UpArgs a;
  a.x = x; a.w_up = W_up; a.w_gate = W_gate; a.b = b;
  a.M = M; a.d = d_model; a.f = d_ff; a.z_debug = z_debug; a.l1_part = l1_part;
  cudaError_t e = decode_up_eligible(M, d_ff, tile_w) ? launch_up_pack_decode(a, t, sms, s)
                                                       : launch_up_pack(a, t, sms, s);
  if (e != cudaSuccess) return TWELL_ERR_CUDA;
  e = launch_overflow_finalize(t, s);
  if (e != cudaSuccess) return TWELL_ERR_CUDA;
  if (l1 == nullptr && nnz_row == nullptr) return TWELL_OK;
  return from_cuda(launch_stats_reduce(t, l1_part, l1, nnz_row, s));
}

twell_status validate_up(const uint16_t *x, const uint16_t *W_up, const uint16_t *W_gate,
                         const uint16_t *b, int M, int d_model, int d_ff, int tile_w, int ell_w,
                         const twell_matrix *out, float *z_debug, void *ws, size_t ws_bytes) {
  twell_status st = check_shape(M, d_ff, tile_w, ell_w);
  if (st != TWELL_OK) return st;
  if (d_model <= 0 || d_model % 64 != 0) return TWELL_ERR_INVALID_ARG;
  if (M == 0) return TWELL_OK;   // documented no-op
  if (x == nullptr || W_up == nullptr || !a16(x) || !a16(W_up) || !a16(W_gate) || !a16(b) ||
      !a16(z_debug))
    return TWELL_ERR_INVALID_ARG;
  st = check_matrix(out, M, d_ff, tile_w, ell_w);
  if (st != TWELL_OK) return st;
  if (ell_w > kMaxEllFused) return TWELL_ERR_UNSUPPORTED;
  if (W_gate != nullptr && tile_w > 128) return TWELL_ERR_UNSUPPORTED;
  return check_ws(ws, ws_bytes, M, d_ff, tile_w, ell_w, out->ovf_capacity);
}

twell_status validate_spmm(const twell_matrix *a, const uint16_t *W_down, int d_model, uint16_t *y,
                           int mode, void *ws, size_t ws_bytes) {
  if (a == nullptr) return TWELL_ERR_INVALID_ARG;
  twell_status st = check_shape(a->M, a->d_ff, a->tile_w, a->ell_w);
  if (st != TWELL_OK) return st;
  if (d_model <= 0 || d_model % 64 != 0) return TWELL_ERR_INVALID_ARG;
  if (mode != TWELL_DOWN_AUTO && mode != TWELL_DOWN_GATHER && mode != TWELL_DOWN_MMA && mode != TWELL_DOWN_SPARSE)
    return TWELL_ERR_INVALID_ARG;
  if (a->M == 0) return TWELL_OK;   // documented no-op
  st = check_matrix(a, a->M, a->d_ff, a->tile_w, a->ell_w);
  if (st != TWELL_OK) return st;
  if (d_model <= 0 || d_model % 64 != 0) return TWELL_ERR_INVALID_ARG;
  if (W_down == nullptr || y == nullptr || !a16(W_down) || !a16(y)) return TWELL_ERR_INVALID_ARG;
  return check_ws(ws, ws_bytes, a->M, a->d_ff, a->tile_w, a->ell_w, a->ovf_capacity, d_model);
}

// pdl_first: the call's first kernel may be a dependent launch (true only when
// the previous kernel on the stream is this library's own, as in
// twell_ffn_forward).  The later kernels of the call always are.
twell_status spmm_checked(const twell_matrix *a, const uint16_t *W_down, int d_model, uint16_t *y,
                          int mode, void *ws, bool pdl_first, cudaStream_t s) {
  if (a->M == 0) return TWELL_OK;
  const TwellView v = make_view(a);
  const int sms = sm_count();
  if (sms <= 0) return TWELL_ERR_CUDA;
  if (mode == TWELL_DOWN_GATHER)
    return from_cuda(launch_spmm_gather(v, W_down, d_model, y, nullptr, pdl_first, s));
  // decode-size batches: the split-K tensor-core kernel streams W_down over every SM
  const Ws w = ws_plan(a->M, a->d_ff, a->tile_w, a->ell_w, a->ovf_capacity, d_model);
  if (decode_down_eligible(a->M)) {
    uint32_t *touch = w.touch_bytes > 0 ? reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(ws) + w.touch) : nullptr;
    return from_cuda(launch_spmm_decode(v, W_down, d_model, y, touch, sms, pdl_first, s));
  }
  int32_t *blk = reinterpret_cast<int32_t *>(static_cast<uint8_t *>(ws) + w.blk_path);
  const SplitWs sp = split_ptrs(w, ws);
  if (mode == TWELL_DOWN_SPARSE && w.sp_bytes > 0) {
    // 2:4 structured-sparse path (explicit mode only: on B200 it measured
    // slower than the dense tensor-core path at every density, see the path's
    // kernel file): the prep pass builds the 2:4 operand and every token's
    // excess product, the decision pass gives each 256-token group its path,
    // and the 2:4 and dense kernels each take their own groups.
    void *spb = static_cast<uint8_t *>(ws) + w.sp;
    cudaError_t e = launch_sp_prep(v, W_down, d_model, spb, -1.0f, true, blk, sp.ctr, pdl_first, s);
    if (e != cudaSuccess) return TWELL_ERR_CUDA;
    e = launch_spmm_sp(v, W_down, d_model, y, blk, spb, sms, true, s);
    if (e != cudaSuccess) return TWELL_ERR_CUDA;
    return from_cuda(launch_spmm_mma(v, W_down, d_model, y, blk, sp, sms, true, s));
  }
  if (mode == TWELL_DOWN_SPARSE) mode = TWELL_DOWN_MMA;   // shape not eligible: dense tensor-core path
  // The block pass also zeroes the split schedule's counters.  MMA mode hands
  // the tensor-core kernel no block flags: its W_down stream starts before the
  // kernel waits for its predecessor, and with no gather launch in between that
  // predecessor is the block pass itself.
  const bool mma_only = mode == TWELL_DOWN_MMA;
  if (!mma_only || sp.ctr != nullptr) {
    cudaError_t e = launch_block_path(v, mma_only ? -1.0f : kDownCrossoverDensity, blk, sp.ctr, pdl_first, s);
    if (e != cudaSuccess) return TWELL_ERR_CUDA;
    pdl_first = true;
  }
  if (!mma_only) {
    cudaError_t e = launch_spmm_gather(v, W_down, d_model, y, blk, true, s);
    if (e != cudaSuccess) return TWELL_ERR_CUDA;
  }
  return from_cuda(launch_spmm_mma(v, W_down, d_model, y, mma_only ? nullptr : blk, sp, sms, pdl_first, s));
}

// Workspace of twell_ffn_backward (every region 256-byte aligned).
struct BwLayout {
  size_t dz_vals, dz_ovf;
  size_t t_vals[2], t_idx[2], t_nnz[2], t_nvf[2], t_pos[2], t_dense[2];   // h^T, dZ^T
  size_t db_part, stage, spmm, total;
  WsLayout stage_L;
};

BwLayout bw_layout(int M, int d_model, int d_ff, int tile_w, int ell_w, int cap, int ell_t, int cap_t) {
  BwLayout b;
  const size_t T = d_ff / tile_w, Tt = M / 128, F = d_ff;
  size_t o = 0;
  auto take = [&](size_t bytes) { const size_t at = o; o = align256(o + bytes); return at; };
  b.dz_vals = take(2 * static_cast<size_t>(M) * T * ell_w);
  b.dz_ovf = take(2 * static_cast<size_t>(cap) * tile_w);
  for (int i = 0; i < 2; ++i) {
    b.t_vals[i] = take(2 * F * Tt * ell_t);
    b.t_idx[i] = take(F * Tt * ell_t);
    b.t_nnz[i] = take(2 * F * Tt);
    b.t_nvf[i] = take(64);
    b.t_pos[i] = take(4 * static_cast<size_t>(cap_t));
    b.t_dense[i] = take(2 * 128 * static_cast<size_t>(cap_t));
  }
  b.db_part = take(4 * F * Tt);
  b.stage_L = ws_layout(d_ff, 128, cap_t);
  b.stage = take(b.stage_L.total);
  const size_t s1 = ws_plan(M, d_ff, tile_w, ell_w, cap, d_model).total,
               s2 = ws_plan(d_ff, M, 128, ell_t, cap_t, d_model).total;
  b.spmm = take(s1 > s2 ? s1 : s2);
  b.total = o;
  return b;
}

// Workspace of twell_spmm_token_overflow (every region 256-byte aligned).
struct TokLayout {
  size_t flag, rank, main_nnz, tok_pos, d_vals, d_idx, d_nnz, y_dense, words, spmm, total;
};

TokLayout tok_layout(int M, int d_model, int d_ff, int tile_w, int ell_w, int cap_tok) {
  TokLayout L;
  const size_t T = d_ff / tile_w;
  size_t o = 0;
  auto take = [&](size_t bytes) { const size_t at = o; o = align256(o + bytes); return at; };
  L.flag = take(4 * static_cast<size_t>(M));
  L.rank = take(4 * static_cast<size_t>(M));
  L.main_nnz = take(2 * static_cast<size_t>(M) * T);
  L.tok_pos = take(4 * static_cast<size_t>(cap_tok));
  L.d_vals = take(2 * static_cast<size_t>(cap_tok) * T * tile_w);
  L.d_idx = take(static_cast<size_t>(cap_tok) * T * tile_w);
  L.d_nnz = take(2 * static_cast<size_t>(cap_tok) * T);
  L.y_dense = take(2 * static_cast<size_t>(cap_tok) * d_model);
  L.words = take(64);
  const size_t s1 = ws_plan(M, d_ff, tile_w, ell_w, 0, d_model).total,
               s2 = ws_plan(cap_tok, d_ff, tile_w, tile_w, 0, d_model).total;
  L.spmm = take(s1 > s2 ? s1 : s2);
  L.total = o;
  return L;
}

}  // namespace

bool a16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool valid_tile(int tile_w) { return tile_w == 32 || tile_w == 64 || tile_w == 128 || tile_w == 256; }

// Shape rules shared by every call.
twell_status check_shape(int M, int d_ff, int tile_w, int ell_w) {
  if (M < 0 || d_ff <= 0 || !valid_tile(tile_w) || d_ff % tile_w != 0) return TWELL_ERR_INVALID_ARG;
  if (ell_w < 1 || ell_w > tile_w) return TWELL_ERR_INVALID_ARG;
  return TWELL_OK;
}

twell_status check_matrix(const twell_matrix *a, int M, int d_ff, int tile_w, int ell_w) {
  if (a == nullptr) return TWELL_ERR_INVALID_ARG;
  if (a->M != M || a->d_ff != d_ff || a->tile_w != tile_w || a->ell_w != ell_w)
    return TWELL_ERR_INVALID_ARG;
  if (a->ovf_capacity < 0 || a->n_ovf == nullptr || a->status == nullptr) return TWELL_ERR_INVALID_ARG;
  if (M > 0 && (a->vals == nullptr || a->idx == nullptr || a->nnz == nullptr)) return TWELL_ERR_INVALID_ARG;
  if (!a16(a->vals) || !a16(a->idx) || !a16(a->nnz)) return TWELL_ERR_INVALID_ARG;
  if (a->ovf_capacity > 0 && (a->ovf_pos == nullptr || a->ovf_dense == nullptr)) return TWELL_ERR_INVALID_ARG;
  if (!a16(a->ovf_pos) || !a16(a->ovf_dense)) return TWELL_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(a->n_ovf) & 3u) || (reinterpret_cast<uintptr_t>(a->status) & 3u))
    return TWELL_ERR_INVALID_ARG;
  return TWELL_OK;
}

twell_status check_pack_args(const uint16_t *h, int M, int d_ff, int ld_h, int tile_w, int ell_w,
                             const twell_matrix *out) {
  twell_status st = check_shape(M, d_ff, tile_w, ell_w);
  if (st != TWELL_OK) return st;
  if (M == 0) return TWELL_OK;   // documented no-op: nothing is read or written
  if (h == nullptr || !a16(h) || ld_h < d_ff || ld_h % 8 != 0) return TWELL_ERR_INVALID_ARG;
  return check_matrix(out, M, d_ff, tile_w, ell_w);
}

CUresult encode_tensor_map_2d(CUtensorMap *map, const void *base, uint64_t inner, uint64_t outer,
                              uint64_t row_pitch_bytes, uint32_t box_inner, uint32_t box_outer,
                              CUtensorMapSwizzle swizzle, CUtensorMapDataType dtype) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return CUDA_ERROR_NOT_INITIALIZED;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_pitch_bytes};
  const cuuint32_t box[2] = {box_inner, box_outer};
  const cuuint32_t elem_strides[2] = {1, 1};
  return fn(map, dtype, 2, const_cast<void *>(base), dims, strides, box,
            elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

CUresult encode_tensor_map_kchunks(CUtensorMap *map, const void *base, uint64_t K, uint64_t rows,
                                   uint32_t box_rows, uint32_t chunks) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return CUDA_ERROR_NOT_INITIALIZED;
  const cuuint64_t dims[3] = {64, rows, K / 64};
  const cuuint64_t strides[2] = {K * 2, 128};   // a row; a 64-element chunk
  const cuuint32_t box[3] = {64, box_rows, chunks};
  const cuuint32_t elem_strides[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box,
            elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

}  // namespace twell

using namespace twell;

extern "C" {

int twell_version(void) { return 300; }

const char *twell_status_string(twell_status s) {
  switch (s) {
    case TWELL_OK: return "ok";
    case TWELL_ERR_INVALID_ARG: return "invalid argument";
    case TWELL_ERR_UNSUPPORTED: return "unsupported configuration";
    case TWELL_ERR_OVERFLOW_CAPACITY: return "overflow backup capacity exhausted";
    case TWELL_ERR_CUDA: return "CUDA error";
    case TWELL_ERR_TIMEOUT: return "device wait timed out";
    case TWELL_ERR_WORKSPACE: return "workspace missing or too small";
  }
  return "unknown status";
}

size_t twell_workspace_bytes(int M, int d_model, int d_ff, int tile_w, int ell_w, int gated,
                             int ovf_capacity) {
  if (check_shape(M, d_ff, tile_w, ell_w) != TWELL_OK || ovf_capacity < 0) return 0;
  if (d_model <= 0 || d_model % 64 != 0 || (gated != 0 && gated != 1)) return 0;
  return ws_plan(M, d_ff, tile_w, ell_w, ovf_capacity, d_model).total;
}

twell_status twell_pack(const uint16_t *h, int M, int d_ff, int ld_h, int tile_w, int ell_w,
                        const twell_matrix *out, void *ws, size_t ws_bytes, void *stream) {
  twell_status st = check_pack_args(h, M, d_ff, ld_h, tile_w, ell_w, out);
  if (st != TWELL_OK || M == 0) return st;
  st = check_ws(ws, ws_bytes, M, d_ff, tile_w, ell_w, out->ovf_capacity);
  if (st != TWELL_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const PackTarget t = make_target(out, ws);
  st = reset_for_pack(t, s);
  if (st != TWELL_OK) return st;
  if (launch_pack_dense(h, ld_h, t, s) != cudaSuccess) return TWELL_ERR_CUDA;
  return from_cuda(launch_overflow_finalize(t, s));
}

twell_status twell_up_pack(const uint16_t *x, const uint16_t *W_up, const uint16_t *W_gate,
                           const uint16_t *b, int M, int d_model, int d_ff, int tile_w, int ell_w,
                           const twell_matrix *out, float *z_debug, void *ws, size_t ws_bytes,
                           void *stream) {
  twell_status st = validate_up(x, W_up, W_gate, b, M, d_model, d_ff, tile_w, ell_w, out, z_debug,
                                ws, ws_bytes);
  if (st != TWELL_OK) return st;
  return up_pack_checked(x, W_up, W_gate, b, M, d_model, d_ff, tile_w, ell_w, out, z_debug, ws,
                         ws_bytes, static_cast<cudaStream_t>(stream));
}

twell_status twell_up_pack_stats(const uint16_t *x, const uint16_t *W_up, const uint16_t *W_gate,
                                 const uint16_t *b, int M, int d_model, int d_ff, int tile_w,
                                 int ell_w, const twell_matrix *out, float *l1, int32_t *nnz_row,
                                 void *ws, size_t ws_bytes, void *stream) {
  twell_status st = validate_up(x, W_up, W_gate, b, M, d_model, d_ff, tile_w, ell_w, out, nullptr,
                                ws, ws_bytes);
  if (st != TWELL_OK) return st;
  if (M > 0 && (!a16(l1) || !a16(nnz_row))) return TWELL_ERR_INVALID_ARG;
  return up_pack_checked(x, W_up, W_gate, b, M, d_model, d_ff, tile_w, ell_w, out, nullptr, ws,
                         ws_bytes, static_cast<cudaStream_t>(stream), l1, nnz_row);
}

twell_status twell_spmm(const twell_matrix *a, const uint16_t *W_down, int d_model, uint16_t *y,
                        int mode, void *ws, size_t ws_bytes, void *stream) {
  twell_status st = validate_spmm(a, W_down, d_model, y, mode, ws, ws_bytes);
  if (st != TWELL_OK) return st;
  return spmm_checked(a, W_down, d_model, y, mode, ws, false, static_cast<cudaStream_t>(stream));
}

twell_status twell_ffn_forward(const uint16_t *x, const uint16_t *W_up, const uint16_t *W_gate,
                               const uint16_t *b, const uint16_t *W_down, int M, int d_model,
                               int d_ff, int tile_w, int ell_w, const twell_matrix *twell, uint16_t *y,
                               int mode, void *ws, size_t ws_bytes, void *stream) {
  twell_status st = validate_up(x, W_up, W_gate, b, M, d_model, d_ff, tile_w, ell_w, twell, nullptr,
                                ws, ws_bytes);
  if (st != TWELL_OK) return st;
  st = validate_spmm(twell, W_down, d_model, y, mode, ws, ws_bytes);
  if (st != TWELL_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  st = up_pack_checked(x, W_up, W_gate, b, M, d_model, d_ff, tile_w, ell_w, twell, nullptr, ws,
                       ws_bytes, s);
  if (st != TWELL_OK) return st;
  // the down kernels follow this call's own producer: dependent launches throughout
  return spmm_checked(twell, W_down, d_model, y, mode, ws, true, s);
}

size_t twell_backward_workspace_bytes(int M, int d_model, int d_ff, int tile_w, int ell_w,
                                      int ovf_capacity, int ell_w_t, int ovf_capacity_t) {
  if (check_shape(M, d_ff, tile_w, ell_w) != TWELL_OK || ovf_capacity < 0 || ovf_capacity_t < 0) return 0;
  if (d_model <= 0 || d_model % 64 != 0 || M % 128 != 0 || d_ff % 128 != 0 || tile_w > 128) return 0;
  if (ell_w_t < 1 || ell_w_t > 128) return 0;
  return bw_layout(M, d_model, d_ff, tile_w, ell_w, ovf_capacity, ell_w_t, ovf_capacity_t).total;
}

twell_status twell_ffn_backward(const uint16_t *x, const uint16_t *W_up, const uint16_t *W_down,
                                const twell_matrix *h, const uint16_t *dY, int d_model, int ell_w_t,
                                int ovf_capacity_t, uint16_t *dX, uint16_t *dW_up, float *db,
                                uint16_t *dW_down, void *ws, size_t ws_bytes, void *stream) {
  if (h == nullptr) return TWELL_ERR_INVALID_ARG;
  twell_status st = check_shape(h->M, h->d_ff, h->tile_w, h->ell_w);
  if (st != TWELL_OK) return st;
  const int M = h->M, f = h->d_ff, tw = h->tile_w, E = h->ell_w;
  if (d_model <= 0 || d_model % 64 != 0) return TWELL_ERR_INVALID_ARG;
  if (M % 128 != 0 || f % 128 != 0 || tw > 128) return TWELL_ERR_UNSUPPORTED;
  if (ell_w_t < 1 || ell_w_t > 128 || ovf_capacity_t < 0) return TWELL_ERR_INVALID_ARG;
  if (M == 0) return TWELL_OK;
  st = check_matrix(h, M, f, tw, E);
  if (st != TWELL_OK) return st;
  const void *ptrs[] = {x, W_up, W_down, dY, dX, dW_up, db, dW_down};
  for (const void *q : ptrs)
    if (q == nullptr || !a16(q)) return TWELL_ERR_INVALID_ARG;
  const BwLayout L = bw_layout(M, d_model, f, tw, E, h->ovf_capacity, ell_w_t, ovf_capacity_t);
  if (ws == nullptr || !a16(ws) || ws_bytes < L.total) return TWELL_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int sms = sm_count();
  if (sms <= 0) return TWELL_ERR_CUDA;
  uint8_t *base = static_cast<uint8_t *>(ws);
  void *spmm_ws = base + L.spmm;

  // 1. dZ at the forward's pattern; it shares the forward's indices, counts
  //    and backup positions
  const TwellView hv = make_view(h);
  uint16_t *dz_vals = reinterpret_cast<uint16_t *>(base + L.dz_vals);
  uint16_t *dz_ovf = reinterpret_cast<uint16_t *>(base + L.dz_ovf);
  if (launch_sddmm(hv, dY, W_down, d_model, dz_vals, dz_ovf, sms, s) != cudaSuccess) return TWELL_ERR_CUDA;
  twell_matrix dz = *h;
  dz.vals = dz_vals;
  dz.ovf_dense = dz_ovf;
  // 2. dX = dZ W_up
  st = spmm_checked(&dz, W_up, d_model, dX, TWELL_DOWN_AUTO, spmm_ws, true, s);
  if (st != TWELL_OK) return st;

  // 3./5. h^T and dZ^T (tiles of 128 tokens); 4./6. dW_down = h^T dY, dW_up = dZ^T x
  const twell_matrix *src[2] = {h, &dz};
  const uint16_t *rhs[2] = {dY, x};
  uint16_t *outw[2] = {dW_down, dW_up};
  for (int i = 0; i < 2; ++i) {
    twell_matrix tm;
    tm.M = f; tm.d_ff = M; tm.tile_w = 128; tm.ell_w = ell_w_t;
    tm.vals = reinterpret_cast<uint16_t *>(base + L.t_vals[i]);
    tm.idx = base + L.t_idx[i];
    tm.nnz = reinterpret_cast<uint16_t *>(base + L.t_nnz[i]);
    tm.ovf_capacity = ovf_capacity_t;
    tm.n_ovf = reinterpret_cast<int32_t *>(base + L.t_nvf[i]);
    tm.ovf_pos = reinterpret_cast<int32_t *>(base + L.t_pos[i]);
    tm.ovf_dense = reinterpret_cast<uint16_t *>(base + L.t_dense[i]);
    tm.status = h->status;   // asynchronous errors land in the forward matrix's word
    PackTarget t;
    t.M = f; t.f = M; t.tw = 128; t.E = ell_w_t; t.T = M / 128;
    t.vals = tm.vals; t.idx = tm.idx; t.nnz = tm.nnz;
    t.cap = ovf_capacity_t; t.n_ovf = tm.n_ovf; t.ovf_pos = tm.ovf_pos; t.ovf_dense = tm.ovf_dense;
    t.status = h->status;
    t.stage_ctr = reinterpret_cast<int32_t *>(base + L.stage + L.stage_L.ctr);
    t.row_ovf = reinterpret_cast<int32_t *>(base + L.stage + L.stage_L.row_ovf);
    t.row_prefix = reinterpret_cast<int32_t *>(base + L.stage + L.stage_L.row_prefix);
    t.stage_pos = reinterpret_cast<int32_t *>(base + L.stage + L.stage_L.stage_pos);
    t.stage_dense = reinterpret_cast<uint16_t *>(base + L.stage + L.stage_L.stage_dense);
    const size_t clr = reinterpret_cast<uint8_t *>(t.row_ovf + f) - reinterpret_cast<uint8_t *>(t.stage_ctr);
    if (cudaMemsetAsync(t.stage_ctr, 0, clr, s) != cudaSuccess) return TWELL_ERR_CUDA;
    float *part = (i == 1) ? reinterpret_cast<float *>(base + L.db_part) : nullptr;
    if (launch_twell_transpose(make_view(src[i]), t, part, false, s) != cudaSuccess) return TWELL_ERR_CUDA;
    if (launch_overflow_finalize(t, s) != cudaSuccess) return TWELL_ERR_CUDA;
    if (i == 1 && launch_stats_reduce(t, part, db, nullptr, s) != cudaSuccess) return TWELL_ERR_CUDA;
    st = spmm_checked(&tm, rhs[i], d_model, outw[i], TWELL_DOWN_AUTO, spmm_ws, true, s);
    if (st != TWELL_OK) return st;
  }
  return TWELL_OK;
}

size_t twell_token_overflow_workspace_bytes(int M, int d_model, int d_ff, int tile_w, int ell_w,
                                            int cap_tok) {
  if (check_shape(M, d_ff, tile_w, ell_w) != TWELL_OK || cap_tok < 1) return 0;
  if (d_model <= 0 || d_model % 64 != 0) return 0;
  return tok_layout(M, d_model, d_ff, tile_w, ell_w, cap_tok).total;
}

twell_status twell_spmm_token_overflow(const twell_matrix *a, const uint16_t *W_down, int d_model,
                                       uint16_t *y, int cap_tok, int32_t *n_tok, void *ws,
                                       size_t ws_bytes, void *stream) {
  if (a == nullptr || cap_tok < 1) return TWELL_ERR_INVALID_ARG;
  twell_status st = check_shape(a->M, a->d_ff, a->tile_w, a->ell_w);
  if (st != TWELL_OK) return st;
  if (d_model <= 0 || d_model % 64 != 0) return TWELL_ERR_INVALID_ARG;
  if (a->M == 0) return TWELL_OK;
  st = check_matrix(a, a->M, a->d_ff, a->tile_w, a->ell_w);
  if (st != TWELL_OK) return st;
  if (W_down == nullptr || y == nullptr || !a16(W_down) || !a16(y) || !a16(n_tok))
    return TWELL_ERR_INVALID_ARG;
  const int M = a->M, f = a->d_ff, tw = a->tile_w;
  const TokLayout L = tok_layout(M, d_model, f, tw, a->ell_w, cap_tok);
  if (ws == nullptr || !a16(ws) || ws_bytes < L.total) return TWELL_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t *base = static_cast<uint8_t *>(ws);
  int32_t *words = reinterpret_cast<int32_t *>(base + L.words);   // [0] zero n_ovf, [1] n_tok
  int32_t *ntok = n_tok != nullptr ? n_tok : words + 1;
  if (cudaMemsetAsync(words, 0, 64, s) != cudaSuccess) return TWELL_ERR_CUDA;
  const TwellView av = make_view(a);
  int32_t *flag = reinterpret_cast<int32_t *>(base + L.flag);
  int32_t *rank = reinterpret_cast<int32_t *>(base + L.rank);
  if (launch_tok_flags(av, flag, s) != cudaSuccess) return TWELL_ERR_CUDA;
  PackTarget scan = {};
  scan.M = M; scan.row_ovf = flag; scan.row_prefix = rank; scan.n_ovf = ntok; scan.cap = cap_tok;
  scan.status = a->status;
  if (launch_row_scan(scan, true, s) != cudaSuccess) return TWELL_ERR_CUDA;
  uint16_t *main_nnz = reinterpret_cast<uint16_t *>(base + L.main_nnz);
  int32_t *tok_pos = reinterpret_cast<int32_t *>(base + L.tok_pos);
  twell_matrix dm;   // the overflowing tokens' rows, ell_w = tile_w
  dm.M = cap_tok; dm.d_ff = f; dm.tile_w = tw; dm.ell_w = tw;
  dm.vals = reinterpret_cast<uint16_t *>(base + L.d_vals);
  dm.idx = base + L.d_idx;
  dm.nnz = reinterpret_cast<uint16_t *>(base + L.d_nnz);
  dm.ovf_capacity = 0; dm.n_ovf = words; dm.ovf_pos = nullptr; dm.ovf_dense = nullptr;
  dm.status = a->status;
  if (launch_tok_build(av, flag, rank, ntok, cap_tok, main_nnz, tok_pos, dm.vals, dm.idx, dm.nnz, s) != cudaSuccess)
    return TWELL_ERR_CUDA;
  twell_matrix mm = *a;   // the other tokens: their slots, no backup
  mm.nnz = main_nnz;
  mm.ovf_capacity = 0; mm.n_ovf = words; mm.ovf_pos = nullptr; mm.ovf_dense = nullptr;
  void *spmm_ws = base + L.spmm;
  st = spmm_checked(&mm, W_down, d_model, y, TWELL_DOWN_AUTO, spmm_ws, true, s);
  if (st != TWELL_OK) return st;
  uint16_t *y_dense = reinterpret_cast<uint16_t *>(base + L.y_dense);
  st = spmm_checked(&dm, W_down, d_model, y_dense, TWELL_DOWN_AUTO, spmm_ws, true, s);
  if (st != TWELL_OK) return st;
  return from_cuda(launch_tok_scatter(ntok, cap_tok, tok_pos, y_dense, d_model, y, s));
}

twell_status twell_read_status(const twell_matrix *a, void *stream, int32_t *n_ovf_out) {
  if (a == nullptr || a->status == nullptr || a->n_ovf == nullptr) return TWELL_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return TWELL_ERR_CUDA;
  int32_t st = 0, n = 0;
  if (cudaMemcpy(&st, a->status, sizeof(st), cudaMemcpyDeviceToHost) != cudaSuccess) return TWELL_ERR_CUDA;
  if (cudaMemcpy(&n, a->n_ovf, sizeof(n), cudaMemcpyDeviceToHost) != cudaSuccess) return TWELL_ERR_CUDA;
  if (n_ovf_out) *n_ovf_out = n;
  return static_cast<twell_status>(st);
}

}  // extern "C"
