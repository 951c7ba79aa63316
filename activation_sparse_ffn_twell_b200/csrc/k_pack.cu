// TwELL packing of a dense bf16 hidden matrix, and the overflow finaliser that
// turns the unordered staged backup into the canonical ascending list.
//
// TwELL (upppp.jp 2026-05-11, section 「TwELLとカスタムCUDAカーネルが解決する課題」):
// hidden columns are cut into tiles of tile_w; per (token, tile) the nonzeros are
// kept as ELL slots (value, in-tile index) in ascending column order; a pair with
// more than ell_w nonzeros also keeps its dense segment in the backup.
//
// Packing is HBM-bound (read h once, write the packed form once): one warp per
// (token, tile) pair, lanes own contiguous column groups so the read is a single
// coalesced segment, and slot positions come from warp ballots + popcounts.
#include "twell_device.cuh"

namespace twell {
namespace {

template <int TW>
__global__ void __launch_bounds__(256) k_pack_dense(const uint16_t *__restrict__ h, int ld_h,
                                                    PackTarget p) {
  griddep_launch_dependents();   // the backup scan waits for this grid anyway
  griddep_wait();                // the call's reset kernel
  constexpr int EPL = TW / 32;  // elements per lane (1, 2, 4, 8)
  const int lane = threadIdx.x & 31;
  const int warps_per_cta = blockDim.x >> 5;
  const long long n_pairs = static_cast<long long>(p.M) * p.T;
  const unsigned full = 0xFFFFFFFFu;
  const unsigned lt_mask = (1u << lane) - 1u;

  for (long long pair = static_cast<long long>(blockIdx.x) * warps_per_cta + (threadIdx.x >> 5);
       pair < n_pairs; pair += static_cast<long long>(gridDim.x) * warps_per_cta) {
    const int r = static_cast<int>(pair / p.T);
    const int t = static_cast<int>(pair - static_cast<long long>(r) * p.T);
    const uint16_t *src = h + static_cast<size_t>(r) * ld_h + static_cast<size_t>(t) * TW + lane * EPL;

    uint16_t v[EPL];
    if constexpr (EPL == 8) {
      uint4 q = __ldg(reinterpret_cast<const uint4 *>(src));
      const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) { v[2 * i] = w[i] & 0xFFFF; v[2 * i + 1] = w[i] >> 16; }
    } else if constexpr (EPL == 4) {
      uint2 q = __ldg(reinterpret_cast<const uint2 *>(src));
      v[0] = q.x & 0xFFFF; v[1] = q.x >> 16; v[2] = q.y & 0xFFFF; v[3] = q.y >> 16;
    } else if constexpr (EPL == 2) {
      uint32_t q = __ldg(reinterpret_cast<const unsigned int *>(src));
      v[0] = q & 0xFFFF; v[1] = q >> 16;
    } else {
      v[0] = __ldg(src);
    }

    // rank of each nonzero among the pair's nonzeros in ascending column order
    int before = 0;   // nonzeros in lanes below this one
    int total = 0;
    unsigned nzbits = 0;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      const bool nz = (v[i] & 0x7FFF) != 0;
      nzbits |= (nz ? 1u : 0u) << i;
      const unsigned m = __ballot_sync(full, nz);
      before += __popc(m & lt_mask);
      total += __popc(m);
    }
    const size_t rec = static_cast<size_t>(pair) * p.E;
    int rank = before;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      if ((nzbits >> i) & 1u) {
        if (rank < p.E) {
          p.vals[rec + rank] = v[i];
          p.idx[rec + rank] = static_cast<uint8_t>(lane * EPL + i);
        }
        ++rank;
      }
    }
    for (int s = total + lane; s < p.E; s += 32) {   // padding slots: (+0, 0)
      p.vals[rec + s] = 0;
      p.idx[rec + s] = 0;
    }
    if (lane == 0) p.nnz[pair] = static_cast<uint16_t>(total);

    if (total > p.E) {   // warp-uniform: stage the dense segment
      int k = 0;
      if (lane == 0) {
        k = atomicAdd(p.stage_ctr, 1);
        atomicAdd(p.row_ovf + r, 1);
        if (k < p.cap) p.stage_pos[k] = static_cast<int32_t>(pair);
      }
      k = __shfl_sync(full, k, 0);
      if (k < p.cap) {
        uint16_t *dst = p.stage_dense + static_cast<size_t>(k) * TW + lane * EPL;
#pragma unroll
        for (int i = 0; i < EPL; ++i) dst[i] = ((v[i] & 0x7FFF) != 0) ? v[i] : 0;
      }
    }
  }
}

// Exclusive scan of the per-token overflow counts (one CTA, any M), total ->
// n_ovf, capacity check -> status.
__global__ void __launch_bounds__(1024) k_ovf_row_scan(PackTarget p) {
  // each thread owns 8 consecutive rows per round of 8192 (one round up to
  // M = 8192): two 16-byte loads, a local scan, one block scan of the totals
  __shared__ int warp_sums[32];
  __shared__ int carry_s;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  griddep_launch_dependents();
  griddep_wait();   // the producer's counts
  int carry = 0;
  for (int base = 0; base < p.M; base += 1024 * 8) {
    const int i0 = base + tid * 8;
    int v[8];
    if (i0 + 8 <= p.M) {   // the count array is 256-byte aligned: i0 * 4 is 32-byte aligned
      const int4 a = reinterpret_cast<const int4 *>(p.row_ovf + i0)[0];
      const int4 b = reinterpret_cast<const int4 *>(p.row_ovf + i0)[1];
      v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) v[j] = (i0 + j < p.M) ? p.row_ovf[i0 + j] : 0;
    }
    int tot = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) tot += v[j];
    int incl = tot;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xFFFFFFFFu, incl, o);
      if (lane >= o) incl += n;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      int ws = warp_sums[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xFFFFFFFFu, ws, o);
        if (lane >= o) ws += n;
      }
      warp_sums[lane] = ws;   // inclusive over warps
      if (lane == 31) carry_s = ws;
    }
    __syncthreads();
    int run = carry + (warp ? warp_sums[warp - 1] : 0) + incl - tot;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (i0 + j < p.M) p.row_prefix[i0 + j] = run;
      run += v[j];
    }
    carry += carry_s;
    __syncthreads();   // warp_sums / carry_s are rewritten by the next pass of the loop
  }
  if (tid == 0) {
    *p.n_ovf = carry;
    if (carry > p.cap) raise_status(p.status, TWELL_ERR_OVERFLOW_CAPACITY);
  }
}

// Move each staged segment to its rank in the ascending r*T+t order.
template <int TW>
__global__ void __launch_bounds__(256) k_ovf_scatter(PackTarget p) {
  griddep_launch_dependents();
  griddep_wait();   // the row prefix
  const int lane = threadIdx.x & 31;
  const int warps_per_cta = blockDim.x >> 5;
  const int staged = min(*p.stage_ctr, p.cap);
  for (int k = blockIdx.x * warps_per_cta + (threadIdx.x >> 5); k < staged;
       k += gridDim.x * warps_per_cta) {
    const int pos = p.stage_pos[k];
    const int r = pos / p.T, t = pos - r * p.T;
    int before = 0;
    for (int t0 = 0; t0 < t; t0 += 32) {
      const int tt = t0 + lane;
      const bool ov = (tt < t) && (static_cast<int>(p.nnz[static_cast<size_t>(r) * p.T + tt]) > p.E);
      before += __popc(__ballot_sync(0xFFFFFFFFu, ov));
    }
    const int rank = p.row_prefix[r] + before;
    if (rank >= p.cap) continue;
    if (lane == 0) p.ovf_pos[rank] = pos;
    const uint16_t *src = p.stage_dense + static_cast<size_t>(k) * TW;
    uint16_t *dst = p.ovf_dense + static_cast<size_t>(rank) * TW;
    constexpr int kVec = TW / 8;   // 16-byte vectors per segment (4 .. 32)
    for (int c = lane; c < kVec; c += 32)
      reinterpret_cast<uint4 *>(dst)[c] = reinterpret_cast<const uint4 *>(src)[c];
  }
}

// Batches of at most kSmallScanRows tokens: the backup scan and the scatter in
// one kernel.  Every CTA loads the per-token overflow counts into shared memory
// and scans them (one warp, 8 tokens per lane); CTA 0 also writes n_ovf and the
// capacity status.  Then each warp moves its staged segments as k_ovf_scatter.
constexpr int kSmallScanRows = 256;

template <int TW>
__global__ void __launch_bounds__(256) k_ovf_finalize_small(PackTarget p) {
  __shared__ int prefix_s[kSmallScanRows];
  griddep_launch_dependents();
  griddep_wait();   // the producer's counts and staged segments
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (warp == 0) {
    int v[8], tot = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int r = lane * 8 + j;
      v[j] = r < p.M ? p.row_ovf[r] : 0;
      tot += v[j];
    }
    int incl = tot;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xFFFFFFFFu, incl, o);
      if (lane >= o) incl += n;
    }
    int run = incl - tot;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      prefix_s[lane * 8 + j] = run;
      run += v[j];
    }
    if (blockIdx.x == 0 && lane == 31) {
      *p.n_ovf = incl;
      if (incl > p.cap) raise_status(p.status, TWELL_ERR_OVERFLOW_CAPACITY);
    }
  }
  __syncthreads();
  const int warps_per_cta = blockDim.x >> 5;
  const int staged = min(*p.stage_ctr, p.cap);
  for (int k = blockIdx.x * warps_per_cta + warp; k < staged; k += gridDim.x * warps_per_cta) {
    const int pos = p.stage_pos[k];
    const int r = pos / p.T, t = pos - r * p.T;
    int before = 0;
    for (int t0 = 0; t0 < t; t0 += 32) {
      const int tt = t0 + lane;
      const bool ov = (tt < t) && (static_cast<int>(p.nnz[static_cast<size_t>(r) * p.T + tt]) > p.E);
      before += __popc(__ballot_sync(0xFFFFFFFFu, ov));
    }
    const int rank = prefix_s[r] + before;
    if (rank >= p.cap) continue;
    if (lane == 0) p.ovf_pos[rank] = pos;
    const uint16_t *src = p.stage_dense + static_cast<size_t>(k) * TW;
    uint16_t *dst = p.ovf_dense + static_cast<size_t>(rank) * TW;
    constexpr int kVec = TW / 8;
    for (int c = lane; c < kVec; c += 32)
      reinterpret_cast<uint4 *>(dst)[c] = reinterpret_cast<const uint4 *>(src)[c];
  }
}

// Per token: its tiles' |h| partial sums and TwELL counts added in a fixed
// order (each lane strides the tiles, then a fixed butterfly), so the result
// is the same on every run.
__global__ void __launch_bounds__(256) k_stats_reduce(PackTarget p, const float *l1_part, float *l1,
                                                      int32_t *nnz_row) {
  griddep_wait();   // the producer's partials and counts
  const int lane = threadIdx.x & 31;
  const int warps = blockDim.x >> 5;
  for (int r = blockIdx.x * warps + (threadIdx.x >> 5); r < p.M; r += gridDim.x * warps) {
    const size_t base = static_cast<size_t>(r) * p.T;
    float s = 0.f;
    int c = 0;
    for (int t = lane; t < p.T; t += 32) {
      if (l1_part != nullptr) s += l1_part[base + t];
      c += p.nnz[base + t];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      s += __shfl_xor_sync(0xFFFFFFFFu, s, o);
      c += __shfl_xor_sync(0xFFFFFFFFu, c, o);
    }
    if (lane == 0) {
      if (l1 != nullptr) l1[r] = s;
      if (nnz_row != nullptr) nnz_row[r] = c;
    }
  }
}

int grid_for(long long work_items, int per_cta, int cap_ctas) {
  long long g = (work_items + per_cta - 1) / per_cta;
  if (g < 1) g = 1;
  if (g > cap_ctas) g = cap_ctas;
  return static_cast<int>(g);
}

}  // namespace

cudaError_t launch_pack_dense(const uint16_t *h, int ld_h, const PackTarget &t, cudaStream_t s) {
  const long long pairs = static_cast<long long>(t.M) * t.T;
  if (pairs == 0) return cudaSuccess;
  const int grid = grid_for(pairs, 8, 148 * 64);
  switch (t.tw) {
    case 32: return launch_k(k_pack_dense<32>, dim3(grid), dim3(256), 0, s, true, 1, h, ld_h, t);
    case 64: return launch_k(k_pack_dense<64>, dim3(grid), dim3(256), 0, s, true, 1, h, ld_h, t);
    case 128: return launch_k(k_pack_dense<128>, dim3(grid), dim3(256), 0, s, true, 1, h, ld_h, t);
    case 256: return launch_k(k_pack_dense<256>, dim3(grid), dim3(256), 0, s, true, 1, h, ld_h, t);
    default: return cudaErrorInvalidValue;
  }
}

// The status word and the staging counters of a producer call start at zero.
// The producer that follows is a dependent launch: its loads and MMAs overlap
// this kernel, its writes wait for it.
__global__ void __launch_bounds__(256) k_pack_reset(int32_t *status, int32_t *words, int n) {
  griddep_launch_dependents();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i == 0) *status = 0;
  for (int k = i; k < n; k += gridDim.x * blockDim.x) words[k] = 0;
}

cudaError_t launch_pack_reset(const PackTarget &t, cudaStream_t s) {
  // [stage_ctr, row_ovf + M): the counter, the per-token counts and the padding between
  const int n = static_cast<int>((t.row_ovf + t.M) - t.stage_ctr);
  const int grid = n / 256 + 1 < 148 ? n / 256 + 1 : 148;
  return launch_k(k_pack_reset, dim3(grid), dim3(256), 0, s, false, 1, t.status, t.stage_ctr, n);
}

cudaError_t launch_overflow_finalize(const PackTarget &t, cudaStream_t s) {
  if (t.M == 0) return cudaSuccess;
  if (t.M <= kSmallScanRows) {
    // one dependent launch: the scan of at most 256 counts is repeated per CTA
    const dim3 grid(grid_for(t.cap > 0 ? t.cap : 1, 8, 148 * 8)), block(256);
    switch (t.tw) {
      case 32: return launch_k(k_ovf_finalize_small<32>, grid, block, 0, s, true, 1, t);
      case 64: return launch_k(k_ovf_finalize_small<64>, grid, block, 0, s, true, 1, t);
      case 128: return launch_k(k_ovf_finalize_small<128>, grid, block, 0, s, true, 1, t);
      case 256: return launch_k(k_ovf_finalize_small<256>, grid, block, 0, s, true, 1, t);
      default: return cudaErrorInvalidValue;
    }
  }
  // both follow the producer kernel of the same call: dependent launches
  cudaError_t e = launch_k(k_ovf_row_scan, dim3(1), dim3(1024), 0, s, true, 1, t);
  if (e != cudaSuccess) return e;
  if (t.cap == 0) return cudaSuccess;
  const dim3 grid(grid_for(t.cap, 8, 148 * 8)), block(256);
  switch (t.tw) {
    case 32: return launch_k(k_ovf_scatter<32>, grid, block, 0, s, true, 1, t);
    case 64: return launch_k(k_ovf_scatter<64>, grid, block, 0, s, true, 1, t);
    case 128: return launch_k(k_ovf_scatter<128>, grid, block, 0, s, true, 1, t);
    case 256: return launch_k(k_ovf_scatter<256>, grid, block, 0, s, true, 1, t);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_row_scan(const PackTarget &t, bool pdl, cudaStream_t s) {
  if (t.M == 0) return cudaSuccess;
  return launch_k(k_ovf_row_scan, dim3(1), dim3(1024), 0, s, pdl, 1, t);
}

cudaError_t launch_stats_reduce(const PackTarget &t, const float *l1_part, float *l1, int32_t *nnz_row,
                                cudaStream_t s) {
  if (t.M == 0) return cudaSuccess;
  // follows the backup ordering of the same call: a dependent launch
  return launch_k(k_stats_reduce, dim3(grid_for(t.M, 8, 148 * 8)), dim3(256), 0, s, true, 1, t, l1_part,
                  l1, nnz_row);
}

}  // namespace twell
