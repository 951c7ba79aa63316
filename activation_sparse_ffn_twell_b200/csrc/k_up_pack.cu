// Fused producer of the sparse FFN: dense up (and gate) projection on the
// tcgen05 tensor cores, with the activation and the TwELL packing done in the
// epilogue, so the dense hidden matrix never reaches HBM.
//
// "The inference kernel fuses several matmuls and builds the TwELL
// representation on the fly" (upppp.jp 2026-05-11, section
// 「TwELLとカスタムCUDAカーネルが解決する課題」); the format is aligned to the
// tiles of the tiled matmul so packing adds no memory pass or launch
// (innovatopia.jp, editorial notes).
//
// Design (sm_100a, one CTA per SM, persistent over 128 x 256 accumulator tiles):
//   warp 0      TMA producer: x tile [128 x 64] and weight tile [256 x 64] per
//               stage, 128-byte swizzle, 4-stage ring of mbarriers.
//   warp 1      allocates TMEM (2 accumulators x 256 fp32 columns) and issues
//               tcgen05.mma (M=128, N=256, K=16) from one elected lane.
//   warps 2..5  epilogue: tcgen05.ld the accumulator (thread = token row),
//               bias + ReLU (x up for the gated form), round to bf16, and append
//               nonzeros to the row's ELL slots in shared memory; copy the slots
//               out with 16-byte stores; overflowing (row, tile) pairs re-read
//               their columns from TMEM and stage the dense segment.
// The two TMEM accumulators let the epilogue of tile i overlap the MMAs of
// tile i+1.  Gated layers use N = 2*tile_w: gate rows then up rows of the same
// hidden tile, so one accumulator holds g and u side by side.
#include "twell_device.cuh"

namespace twell {
namespace {

constexpr int kStages = 4;
constexpr int kABytes = kBlockM * kBlockK * 2;   // 16 KB
constexpr int kThreads = 192;

template <int TW, bool GATED>
struct UpCfg {
  static constexpr int N = GATED ? 2 * TW : 256;           // MMA N (accumulator columns)
  static constexpr int TILES_PER_ACC = GATED ? 1 : 256 / TW;
  static constexpr int B_BYTES = N * kBlockK * 2;
  static constexpr int STAGE_BYTES = kABytes + B_BYTES;
  static constexpr uint32_t TMEM_COLS = (2 * N <= 32) ? 32 : (2 * N <= 64) ? 64 : (2 * N <= 128) ? 128 : (2 * N <= 256) ? 256 : 512;
  static constexpr uint32_t IDESC = idesc_bf16_f32(kBlockM, N, 0, 0);
};

struct UpParams {
  const uint16_t *b;
  int M, d, f;
  int num_m_blocks, num_n_blocks, num_kb;
  float *z_debug;
  PackTarget out;
};

__device__ __forceinline__ void load_bias8(const uint16_t *b, int col, float (&bv)[8]) {
  if (b == nullptr) {
#pragma unroll
    for (int i = 0; i < 8; ++i) bv[i] = 0.f;
    return;
  }
  const uint4 q = __ldg(reinterpret_cast<const uint4 *>(b + col));
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) { bv[2 * i] = bf16lo_to_f32(w[i]); bv[2 * i + 1] = bf16hi_to_f32(w[i]); }
}

template <int TW, bool GATED>
__global__ void __launch_bounds__(kThreads, 1)
    k_up_pack(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
              const __grid_constant__ CUtensorMap tmap_g, const UpParams P) {
  using C = UpCfg<TW, GATED>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t *smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);

  uint8_t *sA = smem;                                   // kStages x 16 KB
  uint8_t *sB = smem + kStages * kABytes;               // kStages x B_BYTES
  uint8_t *sSlots = sB + kStages * C::B_BYTES;          // 128 rows of slots
  const int E = P.out.E;
  const int pitch_v = ((2 * E + 15) / 16) * 16 + 16;    // bf16 values (+16 B to spread banks)
  const int pitch_i = ((E + 15) / 16) * 16;             // u8 indices
  uint8_t *sVals = sSlots;
  uint8_t *sIdx = sSlots + kBlockM * pitch_v;
  uint64_t *bars = reinterpret_cast<uint64_t *>(sIdx + kBlockM * pitch_i);   // 2 KB aligned
  uint64_t *full = bars;
  uint64_t *empty = bars + kStages;
  uint64_t *tm_full = bars + 2 * kStages;
  uint64_t *tm_empty = bars + 2 * kStages + 2;
  uint64_t *drain = bars + 2 * kStages + 4;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2 * kStages + 5);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
    for (int i = 0; i < 2; ++i) { mbar_init(&tm_full[i], 1); mbar_init(&tm_empty[i], 4); }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmap_x);
    tma_prefetch_desc(&tmap_w);
    if (GATED) tma_prefetch_desc(&tmap_g);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int num_tiles = P.num_m_blocks * P.num_n_blocks;
  int32_t *status = P.out.status;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0; uint32_t phase = 0;
      uint32_t filled = 0;   // bit i: stage i has been filled at least once
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        const int m_blk = tile % P.num_m_blocks, n_blk = tile / P.num_m_blocks;
        for (int kb = 0; kb < P.num_kb; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) { ok = false; break; }
          mbar_arrive_expect_tx(&full[stage], C::STAGE_BYTES);
          filled |= 1u << stage;
          tma_load_2d(sA + stage * kABytes, &tmap_x, &full[stage], kb * kBlockK, m_blk * kBlockM);
          uint8_t *b_dst = sB + stage * C::B_BYTES;
          if constexpr (GATED) {
            tma_load_2d(b_dst, &tmap_g, &full[stage], kb * kBlockK, n_blk * TW);
            tma_load_2d(b_dst + TW * 128, &tmap_w, &full[stage], kb * kBlockK, n_blk * TW);
          } else {
            tma_load_2d(b_dst, &tmap_w, &full[stage], kb * kBlockK, n_blk * 256);
          }
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) {
        *abort_flag = 1;
        raise_status(status, TWELL_ERR_TIMEOUT);
        // Let issued copies land before the CTA's shared memory goes away: the
        // most recent fill of stage i used phase parity `phase` for stages below
        // the ring position and `phase ^ 1` for the others.
        for (int i = 0; i < kStages; ++i) {
          if (!((filled >> i) & 1u)) continue;
          const uint32_t par = (i < stage) ? phase : (phase ^ 1u);
          mbar_wait_bounded(&full[i], par);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0; uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++it) {
        const int acc = it & 1;
        const uint32_t acc_phase = (it >> 1) & 1;
        if (!mbar_wait(&tm_empty[acc], acc_phase ^ 1u, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * C::N);
        for (int kb = 0; kb < P.num_kb; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + stage * kABytes);
          const uint32_t b_addr = smem_u32(sB + stage * C::B_BYTES);
#pragma unroll
          for (int k = 0; k < kBlockK / kUmmaK; ++k) {
            const uint64_t adesc = smem_desc_sw128(a_addr + k * 32, 16, 1024);
            const uint64_t bdesc = smem_desc_sw128(b_addr + k * 32, 16, 1024);
            umma_bf16(d_tmem, adesc, bdesc, C::IDESC, (kb | k) != 0);
          }
          umma_commit(&empty[stage]);
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma_commit(&tm_full[acc]);
      }
      if (!ok) {
        *abort_flag = 1;
        raise_status(status, TWELL_ERR_TIMEOUT);
      }
      // all issued MMAs must finish before TMEM is released
      umma_commit(drain);
      mbar_wait_bounded(drain, 0);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;                      // TMEM lane quarter of this warp
    const int row_in_tile = q * 32 + lane;
    uint16_t *my_vals = reinterpret_cast<uint16_t *>(sVals + row_in_tile * pitch_v);
    uint8_t *my_idx = sIdx + row_in_tile * pitch_i;
    const PackTarget &O = P.out;
    int it = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++it) {
      const int m_blk = tile % P.num_m_blocks, n_blk = tile / P.num_m_blocks;
      const int acc = it & 1;
      const uint32_t acc_phase = (it >> 1) & 1;
      if (!mbar_wait(&tm_full[acc], acc_phase, abort_flag)) {
        *abort_flag = 1;
        raise_status(status, TWELL_ERR_TIMEOUT);
        break;
      }
      tc_fence_after();
      const int r = m_blk * kBlockM + row_in_tile;
      const bool valid = r < P.M;
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * C::N);

#pragma unroll 1
      for (int u = 0; u < C::TILES_PER_ACC; ++u) {
        const int t = GATED ? n_blk : n_blk * C::TILES_PER_ACC + u;
        if (t >= O.T) break;
        const int col0 = t * TW;                 // first hidden column of the tile
        int cnt = 0;
#pragma unroll 1
        for (int c = 0; c < TW / 32; ++c) {
          // a: pre-activation (gate pre-activation when gated); g: up branch
          uint32_t a[32];
          __syncwarp();
          tmem_ld_32x32b_x32(t_row + u * TW + c * 32, a);
          uint32_t g[GATED ? 32 : 1];
          if constexpr (GATED) tmem_ld_32x32b_x32(t_row + TW + c * 32, g);
          tmem_ld_wait();
          if (P.z_debug != nullptr && valid) {
            float *zr = GATED ? P.z_debug + static_cast<size_t>(r) * 2 * P.f
                              : P.z_debug + static_cast<size_t>(r) * P.f;
#pragma unroll
            for (int j = 0; j < 32; j += 4) {
              *reinterpret_cast<float4 *>(zr + col0 + c * 32 + j) =
                  make_float4(__uint_as_float(a[j]), __uint_as_float(a[j + 1]),
                              __uint_as_float(a[j + 2]), __uint_as_float(a[j + 3]));
              if constexpr (GATED)
                *reinterpret_cast<float4 *>(zr + P.f + col0 + c * 32 + j) =
                    make_float4(__uint_as_float(g[j]), __uint_as_float(g[j + 1]),
                                __uint_as_float(g[j + 2]), __uint_as_float(g[j + 3]));
            }
          }
#pragma unroll
          for (int j8 = 0; j8 < 32; j8 += 8) {
            float bv[8];
            load_bias8(P.b, col0 + c * 32 + j8, bv);
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) {
              const int j = j8 + jj;
              // separately rounded fp32 add / multiply (no contraction), then one
              // bf16 rounding: the arithmetic a test can replay exactly
              float v = fmaxf(__fadd_rn(__uint_as_float(a[j]), bv[jj]), 0.f);
              if constexpr (GATED) v = __fmul_rn(v, __uint_as_float(g[j]));
              const uint32_t hb = bf16_bits_rn(v);
              const bool nz = (hb & 0x7FFFu) != 0;
              if (nz && cnt < E) {
                my_vals[cnt] = static_cast<uint16_t>(hb);
                my_idx[cnt] = static_cast<uint8_t>(c * 32 + j);
              }
              cnt += nz ? 1 : 0;
            }
          }
        }
        if (valid) {
          const size_t pair = static_cast<size_t>(r) * O.T + t;
          O.nnz[pair] = static_cast<uint16_t>(cnt);
          uint16_t *gv = O.vals + pair * E;
          uint8_t *gi = O.idx + pair * E;
          if ((E & 7) == 0) {
            for (int s = 0; s < E; s += 8) {
              uint4 w = *reinterpret_cast<const uint4 *>(my_vals + s);
              uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
              for (int i = 0; i < 4; ++i) {   // slots >= cnt are padding: (+0, 0)
                const int s0 = s + 2 * i;
                if (s0 >= cnt) ww[i] = 0;
                else if (s0 + 1 >= cnt) ww[i] &= 0x0000FFFFu;
              }
              *reinterpret_cast<uint4 *>(gv + s) = make_uint4(ww[0], ww[1], ww[2], ww[3]);
              uint2 iw = *reinterpret_cast<const uint2 *>(my_idx + s);
              uint32_t ib[2] = {iw.x, iw.y};
#pragma unroll
              for (int i = 0; i < 2; ++i) {
                uint32_t m = 0;
#pragma unroll
                for (int bb = 0; bb < 4; ++bb)
                  if (s + 4 * i + bb < cnt) m |= 0xFFu << (8 * bb);
                ib[i] &= m;
              }
              *reinterpret_cast<uint2 *>(gi + s) = make_uint2(ib[0], ib[1]);
            }
          } else {
            for (int s = 0; s < E; ++s) {
              gv[s] = (s < cnt) ? my_vals[s] : static_cast<uint16_t>(0);
              gi[s] = (s < cnt) ? my_idx[s] : static_cast<uint8_t>(0);
            }
          }
        }
        // ---- dense backup for pairs with more nonzeros than slots
        const bool ov = valid && cnt > E;
        if (__any_sync(0xFFFFFFFFu, ov)) {
          int k = -1;
          if (ov) {
            k = atomicAdd(O.stage_ctr, 1);
            atomicAdd(O.row_ovf + r, 1);
            if (k < O.cap) O.stage_pos[k] = r * O.T + t;
          }
          const bool write = ov && k < O.cap;
#pragma unroll 1
          for (int c = 0; c < TW / 32; ++c) {
            uint32_t a[32];
            __syncwarp();
            tmem_ld_32x32b_x32(t_row + u * TW + c * 32, a);
            uint32_t g[GATED ? 32 : 1];
            if constexpr (GATED) tmem_ld_32x32b_x32(t_row + TW + c * 32, g);
            tmem_ld_wait();
            if (write) {
              uint16_t *dst = O.stage_dense + static_cast<size_t>(k) * TW + c * 32;
#pragma unroll
              for (int j8 = 0; j8 < 32; j8 += 8) {
                float bv[8];
                load_bias8(P.b, col0 + c * 32 + j8, bv);
                uint32_t w[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                  uint32_t hb[2];
#pragma unroll
                  for (int e2 = 0; e2 < 2; ++e2) {
                    const int j = j8 + 2 * i + e2;
                    float v = fmaxf(__fadd_rn(__uint_as_float(a[j]), bv[2 * i + e2]), 0.f);
                    if constexpr (GATED) v = __fmul_rn(v, __uint_as_float(g[j]));
                    const uint32_t b16 = bf16_bits_rn(v);
                    hb[e2] = (b16 & 0x7FFFu) ? b16 : 0u;
                  }
                  w[i] = hb[0] | (hb[1] << 16);
                }
                *reinterpret_cast<uint4 *>(dst + j8) = make_uint4(w[0], w[1], w[2], w[3]);
              }
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tm_empty[acc]);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

template <int TW, bool GATED>
size_t up_smem_bytes(int E) {
  using C = UpCfg<TW, GATED>;
  const int pitch_v = ((2 * E + 15) / 16) * 16 + 16;
  const int pitch_i = ((E + 15) / 16) * 16;
  return 1024 + kStages * (kABytes + C::B_BYTES) + kBlockM * (pitch_v + pitch_i) + 64 + 256;
}

template <int TW, bool GATED>
cudaError_t launch_up_impl(const UpArgs &a, const PackTarget &t, int num_sms, cudaStream_t s) {
  using C = UpCfg<TW, GATED>;
  CUtensorMap mx, mw, mg;
  if (encode_tensor_map_2d(&mx, a.x, a.d, a.M, static_cast<uint64_t>(a.d) * 2, kBlockK, kBlockM,
                           CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  const uint32_t w_rows = GATED ? TW : 256;
  if (encode_tensor_map_2d(&mw, a.w_up, a.d, a.f, static_cast<uint64_t>(a.d) * 2, kBlockK, w_rows,
                           CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  if (GATED) {
    if (encode_tensor_map_2d(&mg, a.w_gate, a.d, a.f, static_cast<uint64_t>(a.d) * 2, kBlockK, TW,
                             CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  } else {
    mg = mw;
  }
  UpParams P;
  P.b = a.b;
  P.M = a.M; P.d = a.d; P.f = a.f;
  P.num_m_blocks = (a.M + kBlockM - 1) / kBlockM;
  P.num_n_blocks = GATED ? t.T : (a.f + 255) / 256;
  P.num_kb = a.d / kBlockK;
  P.z_debug = a.z_debug;
  P.out = t;
  const size_t smem = up_smem_bytes<TW, GATED>(t.E);
  cudaError_t e = cudaFuncSetAttribute(k_up_pack<TW, GATED>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int tiles = P.num_m_blocks * P.num_n_blocks;
  const int grid = tiles < num_sms ? tiles : num_sms;
  k_up_pack<TW, GATED><<<grid, kThreads, smem, s>>>(mx, mw, mg, P);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_up_pack(const UpArgs &a, const PackTarget &t, int num_sms, cudaStream_t s) {
  if (a.M == 0) return cudaSuccess;
  const bool gated = a.w_gate != nullptr;
  switch (t.tw) {
    case 32: return gated ? launch_up_impl<32, true>(a, t, num_sms, s) : launch_up_impl<32, false>(a, t, num_sms, s);
    case 64: return gated ? launch_up_impl<64, true>(a, t, num_sms, s) : launch_up_impl<64, false>(a, t, num_sms, s);
    case 128: return gated ? launch_up_impl<128, true>(a, t, num_sms, s) : launch_up_impl<128, false>(a, t, num_sms, s);
    case 256: return gated ? cudaErrorNotSupported : launch_up_impl<256, false>(a, t, num_sms, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace twell
