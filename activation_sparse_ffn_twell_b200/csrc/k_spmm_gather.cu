// Sparse down-projection on CUDA cores: y[r] = sum over the packed nonzeros of
// token r of value * W_down[hidden index], reading only TwELL slots and, for
// overflowing (token, tile) pairs, the dense backup segment.  "The dense
// hidden-by-down product is never run" -- the down projection consumes only the
// packed nonzeros (upppp.jp 2026-05-11, section 「TwELLとカスタムCUDAカーネルが解決する課題」).
//
// Layout: W_down is [d_ff][d_model] so each nonzero reads one contiguous row of
// 2*d_model bytes.  One warp owns one token and a 256*NCH-column slice of y;
// every lane holds 8*NCH fp32 accumulators and reads its 16-byte pieces of the
// gathered row with 128-bit loads (the whole row slice is one coalesced
// request).  Used where a token block is sparse enough that the tensor-core
// path (which rebuilds dense h tiles) would mostly multiply zeros.
#include "twell_device.cuh"

namespace twell {
namespace {

template <int NCH>
__device__ __forceinline__ void fma_row(float (&acc)[NCH][8], const uint16_t *wrow, int col_base,
                                        int d, float v) {
#pragma unroll
  for (int ch = 0; ch < NCH; ++ch) {
    const int col = col_base + ch * 256;
    if (col < d) {
      const uint4 q = __ldg(reinterpret_cast<const uint4 *>(wrow + col));
      const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        acc[ch][2 * i] = fmaf(v, bf16lo_to_f32(w[i]), acc[ch][2 * i]);
        acc[ch][2 * i + 1] = fmaf(v, bf16hi_to_f32(w[i]), acc[ch][2 * i + 1]);
      }
    }
  }
}

// blk_density_ok: NULL, or per 128-token block flag (1 = this path owns the block)
template <int NCH>
__global__ void __launch_bounds__(256) k_spmm_gather(TwellView A, const uint16_t *__restrict__ W,
                                                     int d, uint16_t *__restrict__ y,
                                                     const int32_t *__restrict__ blk_path) {
  griddep_wait();   // TwELL and the block paths of the previous kernels
  const int lane = threadIdx.x & 31;
  const int warps_per_cta = blockDim.x >> 5;
  const int cols_per_pass = 256 * NCH;
  const int passes = (d + cols_per_pass - 1) / cols_per_pass;
  const long long items = static_cast<long long>(A.M) * passes;
  const int n_ovf = min(*A.n_ovf, A.cap);
  const unsigned full = 0xFFFFFFFFu;

  for (long long it = static_cast<long long>(blockIdx.x) * warps_per_cta + (threadIdx.x >> 5);
       it < items; it += static_cast<long long>(gridDim.x) * warps_per_cta) {
    const int r = static_cast<int>(it / passes);
    const int pass = static_cast<int>(it - static_cast<long long>(r) * passes);
    if (blk_path != nullptr && blk_path[r / kBlockM] != kPathGather) continue;   // a tensor-core path's
    const int col_base = pass * cols_per_pass + lane * 8;

    float acc[NCH][8];
#pragma unroll
    for (int ch = 0; ch < NCH; ++ch)
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[ch][i] = 0.f;

    const size_t row_pair0 = static_cast<size_t>(r) * A.T;
    int ovf_base = -1, ovf_seen = 0;
    for (int t0 = 0; t0 < A.T; t0 += 32) {
      const int tt = t0 + lane;
      const int my_n = (tt < A.T) ? static_cast<int>(__ldg(A.nnz + row_pair0 + tt)) : 0;
      unsigned live = __ballot_sync(full, my_n != 0);
      while (live) {
        const int src = __ffs(live) - 1;
        live &= live - 1;
        const int t = t0 + src;
        const int n = __shfl_sync(full, my_n, src);
        const uint16_t *wtile = W + static_cast<size_t>(t) * A.tw * d;
        if (n <= A.E) {
          const size_t rec = (row_pair0 + t) * A.E;
          for (int s0 = 0; s0 < n; s0 += 32) {
            const int s = s0 + lane;
            uint32_t sv = 0, si = 0;
            if (s < n) { sv = __ldg(A.vals + rec + s); si = __ldg(A.idx + rec + s); }
            const int cnt = min(32, n - s0);
            for (int k = 0; k < cnt; ++k) {
              const float v = bf16lo_to_f32(__shfl_sync(full, sv, k));
              const int j = __shfl_sync(full, si, k);
              if (j < A.tw)   // a malformed index must not read past W_down
                fma_row<NCH>(acc, wtile + static_cast<size_t>(j) * d, col_base, d, v);
            }
          }
        } else {
          // this token's backup entries are consecutive: search once, then walk
          if (ovf_base < 0) ovf_base = ovf_lower_bound(A.ovf_pos, n_ovf, r * A.T);
          const int k = ovf_base + ovf_seen++;
          if (k >= n_ovf) continue;   // capacity exhausted: status already raised, y undefined
          const uint16_t *seg = A.ovf_dense + static_cast<size_t>(k) * A.tw;
          for (int j0 = 0; j0 < A.tw; j0 += 32) {
            const uint32_t sv = __ldg(seg + j0 + lane);
            unsigned nzm = __ballot_sync(full, (sv & 0x7FFFu) != 0);
            while (nzm) {
              const int jj = __ffs(nzm) - 1;
              nzm &= nzm - 1;
              const float v = bf16lo_to_f32(__shfl_sync(full, sv, jj));
              fma_row<NCH>(acc, wtile + static_cast<size_t>(j0 + jj) * d, col_base, d, v);
            }
          }
        }
      }
    }
    uint16_t *yr = y + static_cast<size_t>(r) * d;
#pragma unroll
    for (int ch = 0; ch < NCH; ++ch) {
      const int col = col_base + ch * 256;
      if (col < d) {
        uint4 o;
        o.x = pack_bf16x2(acc[ch][0], acc[ch][1]);
        o.y = pack_bf16x2(acc[ch][2], acc[ch][3]);
        o.z = pack_bf16x2(acc[ch][4], acc[ch][5]);
        o.w = pack_bf16x2(acc[ch][6], acc[ch][7]);
        *reinterpret_cast<uint4 *>(yr + col) = o;
      }
    }
  }
}

}  // namespace

cudaError_t launch_spmm_gather(const TwellView &v, const uint16_t *w_down, int d, uint16_t *y,
                               const int32_t *blk_path, bool pdl, cudaStream_t s) {
  if (v.M == 0) return cudaSuccess;
  // widest register tile that keeps every lane busy
  const int nch = (d >= 2048) ? 8 : (d >= 1024) ? 4 : (d >= 512) ? 2 : 1;
  const int passes = (d + 256 * nch - 1) / (256 * nch);
  long long items = static_cast<long long>(v.M) * passes;
  long long grid = (items + 7) / 8;
  if (grid > 148 * 32) grid = 148 * 32;
  if (grid < 1) grid = 1;
  const dim3 g(static_cast<unsigned>(grid)), b(256);
  switch (nch) {
    case 8: return launch_k(k_spmm_gather<8>, g, b, 0, s, pdl, 1, v, w_down, d, y, blk_path);
    case 4: return launch_k(k_spmm_gather<4>, g, b, 0, s, pdl, 1, v, w_down, d, y, blk_path);
    case 2: return launch_k(k_spmm_gather<2>, g, b, 0, s, pdl, 1, v, w_down, d, y, blk_path);
    default: return launch_k(k_spmm_gather<1>, g, b, 0, s, pdl, 1, v, w_down, d, y, blk_path);
  }
}

}  // namespace twell
