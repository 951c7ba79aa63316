// Sparse down-projection on the tcgen05 tensor cores for token blocks whose
// activations are too dense for the CUDA-core gather to win.
//
// The pages' kernels keep sparse data "aligned to the tiles of tiled matmul"
// (innovatopia.jp, editorial notes; upppp.jp 2026-05-11, section
// 「TwELLとカスタムCUDAカーネルが解決する課題」).  Here a 128-token x 64-hidden
// operand tile is rebuilt in shared memory straight from the TwELL slots (plus
// the dense backup segment of overflowing pairs) -- the dense h never exists in
// HBM -- and multiplied by the matching 64 rows of W_down.
//
// Roles (one CTA per SM, persistent over 128-token x 256-column tiles of y):
//   warp 0      TMA: W_down[k0:k0+64, n0:n0+256] as four 64x64 boxes, 128-byte
//               swizzle; this is an N-major ("MN-major") B operand.
//   warp 1      TMEM allocation (2 x 256 fp32 columns) + tcgen05.mma issue.
//   warps 2..5  epilogue: TMEM -> fp32 registers -> bf16 -> y.
//   warps 6..9  A builders: thread = token row.  Fast path (ell_w % 8 == 0):
//               the row's slot record of the next hidden tile is loaded into
//               registers with 128/64-bit loads while the current one is used;
//               the K steps of one tile are claimed together, zeroed with
//               bank-conflict-free 16-byte stores, and each slot is written once
//               with a predicated 2-byte store (fully unrolled over ell_w).
//               General path: per K step, zero the row and scatter from global
//               memory.  Then fence to the async proxy and arrive.
#include "twell_device.cuh"

namespace twell {
namespace {

constexpr int kMaxStages = 4;
constexpr int kBN = 256;                        // y columns per tile
constexpr int kABytes = kBlockM * kBlockK * 2;  // 16 KB
constexpr int kBBytes = kBlockK * kBN * 2;      // 32 KB (4 boxes of 64 x 64)
constexpr int kThreads = 320;
constexpr uint32_t kIdesc = idesc_bf16_f32(kBlockM, kBN, 0, 1);   // A K-major, B N-major

struct DownParams {
  TwellView A;
  uint16_t *y;
  int d;
  int num_m_blocks, num_n_blocks, num_kb;
  int stages;                // pipeline depth (<= kMaxStages), set from shared-memory budget
  const int32_t *blk_path;   // NULL, or per 128-token block: 1 = this path owns it
};

__device__ __forceinline__ int find_ovf(const int32_t *pos, int n, int key) {
  int lo = 0, hi = n - 1;
  while (lo <= hi) {
    const int mid = (lo + hi) >> 1;
    const int v = __ldg(pos + mid);
    if (v == key) return mid;
    if (v < key) lo = mid + 1; else hi = mid - 1;
  }
  return -1;
}

__device__ __forceinline__ bool tile_owned(const DownParams &P, int m_blk) {
  return P.blk_path == nullptr || P.blk_path[m_blk] != 0;
}

template <int EV>   // ell_w / 8 on the fast builder path, 0 = general path
__global__ void __launch_bounds__(kThreads, 1)
    k_spmm_mma(const __grid_constant__ CUtensorMap tmap_wd, const DownParams P) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t *smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  const int kStages = P.stages;
  uint8_t *sA = smem;
  uint8_t *sB = smem + kStages * kABytes;
  uint64_t *bars = reinterpret_cast<uint64_t *>(sB + kStages * kBBytes);
  uint64_t *full = bars;
  uint64_t *empty = bars + kMaxStages;
  uint64_t *tm_full = bars + 2 * kMaxStages;
  uint64_t *tm_empty = bars + 2 * kMaxStages + 2;
  uint64_t *drain = bars + 2 * kMaxStages + 4;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2 * kMaxStages + 5);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const TwellView &A = P.A;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) { mbar_init(&full[i], 1 + 4); mbar_init(&empty[i], 1); }
    for (int i = 0; i < 2; ++i) { mbar_init(&tm_full[i], 1); mbar_init(&tm_empty[i], 4); }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmap_wd);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int num_tiles = P.num_m_blocks * P.num_n_blocks;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA (W_down)
    if (lane == 0) {
      int stage = 0; uint32_t phase = 0; uint32_t filled = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        const int m_blk = tile % P.num_m_blocks, n_blk = tile / P.num_m_blocks;
        if (!tile_owned(P, m_blk)) continue;
        for (int kb = 0; kb < P.num_kb; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) { ok = false; break; }
          mbar_arrive_expect_tx(&full[stage], kBBytes);
          filled |= 1u << stage;
          uint8_t *dst = sB + stage * kBBytes;
#pragma unroll
          for (int j = 0; j < kBN / 64; ++j)
            tma_load_2d(dst + j * (kBlockK * 128), &tmap_wd, &full[stage], n_blk * kBN + j * 64,
                        kb * kBlockK);
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) {
        *abort_flag = 1;
        raise_status(A.status, TWELL_ERR_TIMEOUT);
        for (int i = 0; i < kStages; ++i) {
          if (!((filled >> i) & 1u)) continue;
          mbar_wait_bounded(&full[i], (i < stage) ? phase : (phase ^ 1u));
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0; uint32_t phase = 0; int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        const int m_blk = tile % P.num_m_blocks;
        if (!tile_owned(P, m_blk)) continue;
        const int acc = it & 1;
        const uint32_t acc_phase = (it >> 1) & 1;
        ++it;
        if (!mbar_wait(&tm_empty[acc], acc_phase ^ 1u, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kBN);
        for (int kb = 0; kb < P.num_kb; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + stage * kABytes);
          const uint32_t b_addr = smem_u32(sB + stage * kBBytes);
#pragma unroll
          for (int k = 0; k < kBlockK / kUmmaK; ++k) {
            const uint64_t adesc = smem_desc_sw128(a_addr + k * 32, 16, 1024);
            // N-major B: 16 K-rows of 128 B per step; 64-column groups 8 KB apart
            const uint64_t bdesc = smem_desc_sw128(b_addr + k * 2048, kBlockK * 128, 1024);
            umma_bf16(d_tmem, adesc, bdesc, kIdesc, (kb | k) != 0);
          }
          umma_commit(&empty[stage]);
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma_commit(&tm_full[acc]);
      }
      if (!ok) {
        *abort_flag = 1;
        raise_status(A.status, TWELL_ERR_TIMEOUT);
      }
      umma_commit(drain);
      mbar_wait_bounded(drain, 0);
    }
  } else if (warp < 6) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const int row_in_tile = q * 32 + lane;
    int it = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
      const int m_blk = tile % P.num_m_blocks, n_blk = tile / P.num_m_blocks;
      if (!tile_owned(P, m_blk)) continue;
      const int acc = it & 1;
      const uint32_t acc_phase = (it >> 1) & 1;
      ++it;
      if (!mbar_wait(&tm_full[acc], acc_phase, abort_flag)) {
        *abort_flag = 1;
        raise_status(A.status, TWELL_ERR_TIMEOUT);
        break;
      }
      tc_fence_after();
      const int r = m_blk * kBlockM + row_in_tile;
      const bool valid = r < A.M;
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * kBN);
      uint16_t *yr = P.y + static_cast<size_t>(r) * P.d + n_blk * kBN;
#pragma unroll 1
      for (int c = 0; c < kBN / 32; ++c) {
        uint32_t v[32];
        __syncwarp();
        tmem_ld_32x32b_x32(t_row + c * 32, v);
        tmem_ld_wait();
        if (valid && n_blk * kBN + c * 32 < P.d) {
#pragma unroll
          for (int j = 0; j < 32; j += 8) {
            uint4 o;
            o.x = pack_bf16x2(__uint_as_float(v[j]), __uint_as_float(v[j + 1]));
            o.y = pack_bf16x2(__uint_as_float(v[j + 2]), __uint_as_float(v[j + 3]));
            o.z = pack_bf16x2(__uint_as_float(v[j + 4]), __uint_as_float(v[j + 5]));
            o.w = pack_bf16x2(__uint_as_float(v[j + 6]), __uint_as_float(v[j + 7]));
            *reinterpret_cast<uint4 *>(yr + c * 32 + j) = o;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tm_empty[acc]);
    }
  } else if constexpr (EV > 0) {
    // ------------------------------------------------------------ A builders (fast)
    // ell_w == 8*EV.  Per hidden tile, the row's slot record (values, indices,
    // nnz) is loaded into registers one tile ahead; the tile's K steps are zeroed
    // with independent 16-byte stores and every slot is written once with a
    // predicated 2-byte store -- a fully unrolled, dependency-free sequence.
    constexpr int E = 8 * EV;
    const int row_in_tile = (warp - 6) * 32 + lane;
    const int tw = A.tw, Tn = A.T;
    const int lg_tw = 31 - __clz(tw);
    const int n_ovf = min(*A.n_ovf, A.cap);
    const uint32_t row_swz = static_cast<uint32_t>(row_in_tile & 7);
    int stage = 0; uint32_t phase = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
      const int m_blk = tile % P.num_m_blocks;
      if (!tile_owned(P, m_blk)) continue;
      const int r = m_blk * kBlockM + row_in_tile;
      const bool valid = r < A.M;
      const size_t pair0 = static_cast<size_t>(valid ? r : 0) * Tn;

      // tile t's slot record of this row, straight into registers
      auto fetch = [&](int t, uint4 (&v)[EV], uint2 (&ix)[EV], int &n) {
        if (valid && t < Tn) {
          const uint4 *gv = reinterpret_cast<const uint4 *>(A.vals + (pair0 + t) * E);
          const uint2 *gi = reinterpret_cast<const uint2 *>(A.idx + (pair0 + t) * E);
#pragma unroll
          for (int g = 0; g < EV; ++g) { v[g] = __ldg(gv + g); ix[g] = __ldg(gi + g); }
          n = static_cast<int>(__ldg(A.nnz + pair0 + t));
        } else {
          n = 0;
        }
      };

      int cur_t = -1, n0 = 0, n1 = 0, ovf_k = -1;
      uint4 vq[EV], vq1[EV];
      uint2 iq[EV], iq1[EV];
      // K-steps are claimed in groups of S (all steps of one hidden tile when
      // the ring holds them) so every slot is visited once per tile
      // (at most stages-1 of them, so the MMA always has a stage to work on)
      const int S = max(1, min(tw / kBlockK, kStages - 1));
      for (int kb0 = 0; kb0 < P.num_kb && ok; kb0 += S) {
        const int nsteps = min(S, P.num_kb - kb0);
        const int stage0 = stage;
        for (int j = 0; j < nsteps; ++j) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) { ok = false; break; }
          uint8_t *rowA = sA + stage * kABytes + row_in_tile * 128;
          // Rows are 128 B apart, so lanes storing the same chunk index would all
          // hit the same 4 banks; row-XOR chunk order makes the zeroing conflict-free.
#pragma unroll
          for (int c = 0; c < 8; ++c)
            reinterpret_cast<uint4 *>(rowA)[c ^ static_cast<int>(row_swz)] = make_uint4(0, 0, 0, 0);
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        const int col0 = kb0 * kBlockK, span = nsteps * kBlockK;
        const int t_last = (col0 + span - 1) >> lg_tw;
        for (int t = col0 >> lg_tw; t <= t_last; ++t) {   // 1 tile, or 2 when tile_w == 32
          if (t != cur_t) {                                // same for every thread of the CTA
            if (cur_t < 0) {
              fetch(t, vq, iq, n0);
            } else {
#pragma unroll
              for (int g = 0; g < EV; ++g) { vq[g] = vq1[g]; iq[g] = iq1[g]; }
              n0 = n1;
            }
            fetch(t + 1, vq1, iq1, n1);                    // one tile ahead; used next advance
            cur_t = t;
            ovf_k = (n0 > E) ? find_ovf(A.ovf_pos, n_ovf, static_cast<int>(pair0) + t) : -1;
          }
          if (!valid || t >= Tn || n0 == 0) continue;
          const int base = (t << lg_tw) - col0;           // group column of in-tile index 0
          if (n0 <= E) {
#pragma unroll
            for (int g = 0; g < EV; ++g) {
              const uint32_t vw[4] = {vq[g].x, vq[g].y, vq[g].z, vq[g].w};
              const uint32_t iw[2] = {iq[g].x, iq[g].y};
#pragma unroll
              for (int k = 0; k < 8; ++k) {
                const int sl = 8 * g + k;
                const uint32_t col = static_cast<uint32_t>(base + static_cast<int>((iw[k >> 2] >> (8 * (k & 3))) & 0xFFu));
                if (sl < n0 && col < static_cast<uint32_t>(span)) {
                  int sb = stage0 + static_cast<int>(col >> 6);   // step buffer of this column
                  if (sb >= kStages) sb -= kStages;
                  const uint32_t c = col & 63u;
                  const uint32_t off = (((c >> 3) ^ row_swz) << 4) + ((c & 7u) << 1);
                  *reinterpret_cast<uint16_t *>(sA + sb * kABytes + row_in_tile * 128 + off) =
                      static_cast<uint16_t>((k & 1) ? (vw[k >> 1] >> 16) : (vw[k >> 1] & 0xFFFFu));
                }
              }
            }
          } else if (ovf_k >= 0) {                        // dense backup segment
            // group columns c with in-tile index c - base inside [0, tile_w)
            const int lo = max(0, base), hi = min(span, base + tw);
            for (int c = lo; c < hi; c += 8) {
              const uint4 q = __ldg(reinterpret_cast<const uint4 *>(
                  A.ovf_dense + static_cast<size_t>(ovf_k) * tw + (c - base)));
              int sb = stage0 + (c >> 6);
              if (sb >= kStages) sb -= kStages;
              const uint32_t cc = static_cast<uint32_t>(c & 63);
              *reinterpret_cast<uint4 *>(sA + sb * kABytes + row_in_tile * 128 +
                                         (((cc >> 3) ^ row_swz) << 4)) = q;
            }
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          for (int j = 0; j < nsteps; ++j) {
            int sb = stage0 + j;
            if (sb >= kStages) sb -= kStages;
            mbar_arrive(&full[sb]);
          }
        }
      }
    }
    if (!ok) {
      *abort_flag = 1;
      raise_status(A.status, TWELL_ERR_TIMEOUT);
    }
  } else {
    // ------------------------------------------------------------ A builders (general)
    const int row_in_tile = (warp - 6) * 32 + lane;
    const int n_ovf = min(*A.n_ovf, A.cap);
    int stage = 0; uint32_t phase = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
      const int m_blk = tile % P.num_m_blocks;
      if (!tile_owned(P, m_blk)) continue;
      const int r = m_blk * kBlockM + row_in_tile;
      const bool valid = r < A.M;
      bool ok = true;
      for (int kb = 0; kb < P.num_kb; ++kb) {
        if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) { ok = false; break; }
        uint8_t *tileA = sA + stage * kABytes;
        uint8_t *rowA = tileA + row_in_tile * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c)   // row-XOR chunk order: conflict-free across the warp
          reinterpret_cast<uint4 *>(rowA)[c ^ (row_in_tile & 7)] = make_uint4(0, 0, 0, 0);
        if (valid) {
          const int k0 = kb * kBlockK;               // first hidden column of this stage
          for (int t = k0 / A.tw; t * A.tw < k0 + kBlockK && t < A.T; ++t) {
            const int tc0 = t * A.tw;                 // first hidden column of tile t
            const int lo = max(k0, tc0) - tc0, hi = min(k0 + kBlockK, tc0 + A.tw) - tc0;
            const size_t pair = static_cast<size_t>(r) * A.T + t;
            const int n = __ldg(A.nnz + pair);
            if (n == 0) continue;
            if (n <= A.E) {
              const uint16_t *sv = A.vals + pair * A.E;
              const uint8_t *si = A.idx + pair * A.E;
              for (int s = 0; s < n; ++s) {
                const int j = __ldg(si + s);   // j < tile_w in any valid TwELL
                if (j >= lo && j < hi) {
                  const uint32_t col = static_cast<uint32_t>(tc0 + j - k0);
                  *reinterpret_cast<uint16_t *>(tileA + sw128_offset(row_in_tile, col)) = __ldg(sv + s);
                }
              }
            } else {
              const int k = find_ovf(A.ovf_pos, n_ovf, static_cast<int>(pair));
              if (k < 0) continue;
              const uint16_t *seg = A.ovf_dense + static_cast<size_t>(k) * A.tw;
              for (int j = lo; j < hi; j += 8) {   // 8-column runs are 16-byte aligned
                const uint4 q = __ldg(reinterpret_cast<const uint4 *>(seg + j));
                const uint32_t col = static_cast<uint32_t>(tc0 + j - k0);
                *reinterpret_cast<uint4 *>(tileA + sw128_offset(row_in_tile, col)) = q;
              }
            }
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&full[stage]);
        if (++stage == kStages) { stage = 0; phase ^= 1u; }
      }
      if (!ok) {
        *abort_flag = 1;
        raise_status(A.status, TWELL_ERR_TIMEOUT);
        break;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem_base, 512);
  }
}

// Per 128-token block: 1 when its density is at or above the crossover.
__global__ void __launch_bounds__(256) k_block_path(TwellView A, float crossover, int32_t *blk_path) {
  const int blk = blockIdx.x;
  const int r0 = blk * kBlockM;
  const int rows = min(kBlockM, A.M - r0);
  const long long n = static_cast<long long>(rows) * A.T;
  const uint16_t *base = A.nnz + static_cast<size_t>(r0) * A.T;
  unsigned long long sum = 0;
  for (long long i = threadIdx.x; i < n; i += blockDim.x) sum += __ldg(base + i);
  __shared__ unsigned long long red[256];
  red[threadIdx.x] = sum;
  __syncthreads();
  for (int o = 128; o > 0; o >>= 1) {
    if (threadIdx.x < o) red[threadIdx.x] += red[threadIdx.x + o];
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    const double dens = static_cast<double>(red[0]) / (static_cast<double>(rows) * A.f);
    blk_path[blk] = dens >= crossover ? 1 : 0;
  }
}

template <int EV>
cudaError_t launch_down(const CUtensorMap &mw, const DownParams &P, int grid, size_t smem,
                        cudaStream_t s) {
  cudaError_t e = cudaFuncSetAttribute(k_spmm_mma<EV>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  k_spmm_mma<EV><<<grid, kThreads, smem, s>>>(mw, P);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_block_path(const TwellView &v, float crossover, int32_t *blk_path, cudaStream_t s) {
  const int blocks = (v.M + kBlockM - 1) / kBlockM;
  if (blocks == 0) return cudaSuccess;
  k_block_path<<<blocks, 256, 0, s>>>(v, crossover, blk_path);
  return cudaGetLastError();
}

cudaError_t launch_spmm_mma(const TwellView &v, const uint16_t *w_down, int d, uint16_t *y,
                            const int32_t *blk_path, int num_sms, cudaStream_t s) {
  if (v.M == 0) return cudaSuccess;
  CUtensorMap mw;
  if (encode_tensor_map_2d(&mw, w_down, d, v.f, static_cast<uint64_t>(d) * 2, 64, kBlockK,
                           CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  DownParams P;
  P.A = v;
  P.y = y;
  P.d = d;
  P.num_m_blocks = (v.M + kBlockM - 1) / kBlockM;
  P.num_n_blocks = (d + kBN - 1) / kBN;
  P.num_kb = (v.f + kBlockK - 1) / kBlockK;
  P.blk_path = blk_path;
  const int ev = (v.E % 8 == 0 && v.E <= 64) ? v.E / 8 : 0;
  const size_t fixed = 1024 + 256;
  const size_t budget = 227 * 1024;
  int stages = static_cast<int>((budget - fixed) / (kABytes + kBBytes));
  if (stages > kMaxStages) stages = kMaxStages;
  if (stages < 2) return cudaErrorInvalidValue;
  P.stages = stages;
  const size_t smem = fixed + static_cast<size_t>(stages) * (kABytes + kBBytes);
  const int tiles = P.num_m_blocks * P.num_n_blocks;
  const int grid = tiles < num_sms ? tiles : num_sms;
  switch (ev) {
    case 1: return launch_down<1>(mw, P, grid, smem, s);
    case 2: return launch_down<2>(mw, P, grid, smem, s);
    case 3: return launch_down<3>(mw, P, grid, smem, s);
    case 4: return launch_down<4>(mw, P, grid, smem, s);
    case 5: return launch_down<5>(mw, P, grid, smem, s);
    case 6: return launch_down<6>(mw, P, grid, smem, s);
    case 7: return launch_down<7>(mw, P, grid, smem, s);
    case 8: return launch_down<8>(mw, P, grid, smem, s);
    default: return launch_down<0>(mw, P, grid, smem, s);
  }
}

}  // namespace twell
