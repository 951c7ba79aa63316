// Whole-token overflow form: the alternative reading of the dense backup, in
// which a token with any over-full tile keeps its whole hidden row (stored fully
// dense and run as a small dense product) while the other tokens keep only
// their ELL slots.  Built here from the per-(token, tile) form so the two can be
// compared on the same data; the down-projections are the library's own.
//
//   k_tok_flags   warp per token: 1 if any tile holds more than ell_w nonzeros
//                 (the ascending rank of the flagged tokens comes from the backup
//                 row scan, reused).
//   k_tok_build   warp per (token, tile): the main matrix's count (0 for flagged
//                 tokens) and, for a flagged token, the tile packed with
//                 ell_w = tile_w (every nonzero fits: no backup), from its slots or
//                 its backup segment through a per-warp shared-memory segment.
//   k_tok_scatter the dense tokens' y rows to their places in y.
#include "twell_device.cuh"

namespace twell {
namespace {

__global__ void __launch_bounds__(256) k_tok_flags(TwellView a, int32_t *flag) {
  const int lane = threadIdx.x & 31;
  const int warps = blockDim.x >> 5;
  for (int r = blockIdx.x * warps + (threadIdx.x >> 5); r < a.M; r += gridDim.x * warps) {
    bool over = false;
    for (int t = lane; t < a.T; t += 32) over |= static_cast<int>(__ldg(a.nnz + static_cast<size_t>(r) * a.T + t)) > a.E;
    const bool any = __any_sync(0xFFFFFFFFu, over);
    if (lane == 0) flag[r] = any ? 1 : 0;
  }
}

struct TokBuild {
  TwellView a;
  const int32_t *flag, *rank;   // per token
  const int32_t *n_tok;         // flagged tokens (true count)
  int cap;                      // rows of the dense matrix
  uint16_t *main_nnz;           // [M][T]
  int32_t *tok_pos;             // [cap]
  uint16_t *d_vals;             // [cap][T][tw]
  uint8_t *d_idx;               // [cap][T][tw]
  uint16_t *d_nnz;              // [cap][T]
  int32_t *status;
};

template <int TW>
__global__ void __launch_bounds__(256) k_tok_build(const TokBuild B) {
  constexpr int EPL = TW / 32;
  __shared__ __align__(16) uint16_t seg_all[8][TW];
  griddep_wait();   // the ranks of the scan
  const TwellView &A = B.a;
  const int lane = threadIdx.x & 31, wl = threadIdx.x >> 5;
  uint16_t *seg = seg_all[wl];
  const unsigned lt = (1u << lane) - 1u;
  const int n_ovf = min(*A.n_ovf, A.cap);
  const long long pairs = static_cast<long long>(A.M) * A.T;
  for (long long p = static_cast<long long>(blockIdx.x) * 8 + wl; p < pairs; p += static_cast<long long>(gridDim.x) * 8) {
    const int r = static_cast<int>(p / A.T), t = static_cast<int>(p - static_cast<long long>(r) * A.T);
    const bool flagged = B.flag[r] != 0;
    const int n = __ldg(A.nnz + p);
    if (lane == 0) B.main_nnz[p] = flagged ? 0 : static_cast<uint16_t>(n);
    if (!flagged) continue;
    const int k = B.rank[r];
    if (k >= B.cap) {
      if (lane == 0 && t == 0) raise_status(B.status, TWELL_ERR_OVERFLOW_CAPACITY);
      continue;
    }
    if (lane == 0 && t == 0) B.tok_pos[k] = r;
    // the tile's dense segment, from its slots or its backup segment
    for (int j = lane; j < TW; j += 32) seg[j] = 0;
    __syncwarp();
    if (n <= A.E) {
      for (int s = lane; s < n; s += 32) {
        const int j = __ldg(A.idx + p * A.E + s);
        if (j < TW) seg[j] = __ldg(A.vals + p * A.E + s);
      }
    } else {
      const int kk = ovf_lower_bound(A.ovf_pos, n_ovf, static_cast<int>(p));
      if (kk < n_ovf && __ldg(A.ovf_pos + kk) == static_cast<int>(p))
        for (int j = lane; j < TW; j += 32) seg[j] = __ldg(A.ovf_dense + static_cast<size_t>(kk) * TW + j);
    }
    __syncwarp();
    // packed with ell_w = tile_w: lanes own contiguous columns, ranks by ballot
    uint16_t v[EPL];
    int before = 0, total = 0;
    unsigned bits = 0;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      v[i] = seg[lane * EPL + i];
      const bool nz = (v[i] & 0x7FFFu) != 0;
      bits |= (nz ? 1u : 0u) << i;
      const unsigned m = __ballot_sync(0xFFFFFFFFu, nz);
      before += __popc(m & lt);
      total += __popc(m);
    }
    const size_t rec = (static_cast<size_t>(k) * A.T + t) * TW;
    int rank = before;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      if ((bits >> i) & 1u) {
        B.d_vals[rec + rank] = v[i];
        B.d_idx[rec + rank] = static_cast<uint8_t>(lane * EPL + i);
        ++rank;
      }
    }
    for (int s = total + lane; s < TW; s += 32) { B.d_vals[rec + s] = 0; B.d_idx[rec + s] = 0; }
    if (lane == 0) B.d_nnz[static_cast<size_t>(k) * A.T + t] = static_cast<uint16_t>(total);
    __syncwarp();   // the segment is rewritten by this warp's next pair
  }
}

// Rows of the dense matrix past the flagged tokens: count 0 (their y rows are 0
// and never copied).
__global__ void __launch_bounds__(256) k_tok_clear(const int32_t *n_tok, int cap, int T, uint16_t *d_nnz) {
  griddep_wait();
  const int n = min(*n_tok, cap);
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x + static_cast<long long>(n) * T;
       i < static_cast<long long>(cap) * T; i += static_cast<long long>(gridDim.x) * blockDim.x)
    d_nnz[i] = 0;
}

__global__ void __launch_bounds__(256) k_tok_scatter(const int32_t *n_tok, int cap, const int32_t *tok_pos,
                                                     const uint16_t *y_dense, int d, uint16_t *y) {
  griddep_wait();   // both down-projections
  const int n = min(*n_tok, cap);
  const int per_row = d / 8;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < static_cast<long long>(n) * per_row;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int k = static_cast<int>(i / per_row), c = static_cast<int>(i - static_cast<long long>(k) * per_row);
    reinterpret_cast<uint4 *>(y + static_cast<size_t>(tok_pos[k]) * d)[c] =
        reinterpret_cast<const uint4 *>(y_dense + static_cast<size_t>(k) * d)[c];
  }
}

int grid_cap(long long items, int per_cta) {
  long long g = (items + per_cta - 1) / per_cta;
  if (g < 1) g = 1;
  if (g > 148 * 16) g = 148 * 16;
  return static_cast<int>(g);
}

}  // namespace

cudaError_t launch_tok_flags(const TwellView &a, int32_t *flag, cudaStream_t s) {
  return launch_k(k_tok_flags, dim3(grid_cap(a.M, 8)), dim3(256), 0, s, false, 1, a, flag);
}

cudaError_t launch_tok_build(const TwellView &a, const int32_t *flag, const int32_t *rank, const int32_t *n_tok,
                             int cap, uint16_t *main_nnz, int32_t *tok_pos, uint16_t *d_vals, uint8_t *d_idx,
                             uint16_t *d_nnz, cudaStream_t s) {
  TokBuild B;
  B.a = a; B.flag = flag; B.rank = rank; B.n_tok = n_tok; B.cap = cap;
  B.main_nnz = main_nnz; B.tok_pos = tok_pos; B.d_vals = d_vals; B.d_idx = d_idx; B.d_nnz = d_nnz;
  B.status = a.status;
  const dim3 g(grid_cap(static_cast<long long>(a.M) * a.T, 8)), b(256);
  cudaError_t e;
  switch (a.tw) {
    case 32: e = launch_k(k_tok_build<32>, g, b, 0, s, true, 1, B); break;
    case 64: e = launch_k(k_tok_build<64>, g, b, 0, s, true, 1, B); break;
    case 128: e = launch_k(k_tok_build<128>, g, b, 0, s, true, 1, B); break;
    case 256: e = launch_k(k_tok_build<256>, g, b, 0, s, true, 1, B); break;
    default: return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess) return e;
  return launch_k(k_tok_clear, dim3(grid_cap(static_cast<long long>(cap) * a.T, 256)), dim3(256), 0, s, true,
                  1, n_tok, cap, a.T, d_nnz);
}

cudaError_t launch_tok_scatter(const int32_t *n_tok, int cap, const int32_t *tok_pos, const uint16_t *y_dense,
                               int d, uint16_t *y, cudaStream_t s) {
  return launch_k(k_tok_scatter, dim3(grid_cap(static_cast<long long>(cap) * (d / 8), 256)), dim3(256), 0, s,
                  true, 1, n_tok, cap, tok_pos, y_dense, d, y);
}

}  // namespace twell
