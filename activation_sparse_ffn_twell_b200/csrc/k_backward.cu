// Backward pass of the non-gated sparse FFN through the forward's TwELL form.
//
// The pages' training kernel runs the whole backward pass without dense matmuls
// on the hybrid sparse-main plus dense-backup representation (upppp.jp
// 2026-05-11, section 「TwELLとカスタムCUDAカーネルが解決する課題」).  Here:
//
//   k_sddmm        dZ = (dY W_down^T) sampled at the forward's nonzero pattern,
//                  on the tcgen05 tensor cores: the GEMM of the forward producer
//                  (dY is the K-major A operand, W_down [d_ff][d_model] the
//                  K-major B operand) with an epilogue that keeps only the
//                  entries the forward packed.  dZ shares the forward's slot
//                  indices, counts and backup positions; its values are new.
//   k_twell_transpose
//                  A [M tokens x d_ff] in TwELL -> A^T [d_ff x M] in TwELL with
//                  tiles of 128 tokens: the layout the weight gradients h^T dY and
//                  dZ^T x are read from by the ordinary sparse down-projection.
//                  Optionally the per-(unit, token tile) sums of the values (for
//                  the bias gradient).
//
// dX = dZ W_up, dW_down = h^T dY and dW_up = dZ^T x then run through the
// library's sparse down-projection unchanged.
#include <cstdlib>

#include "twell_device.cuh"

namespace twell {
namespace {

// ============================================================================ SDDMM
constexpr int kSdThreads = 192;                       // TMA, MMA, 4 epilogue warps
constexpr int kSdN = 256;                             // hidden columns per accumulator
constexpr int kSdStages = 3;
constexpr int kSdABytes = kBlockM * kBlockK * 2;      // dY tile [128 x 64]
constexpr int kSdBBytes = kSdN * kBlockK * 2;         // W_down tile [256 x 64]

struct SddParams {
  int M, d, f;
  int num_m_blocks, num_n_blocks, num_kb;
  TwellView h;            // forward pattern (idx, nnz, backup positions and segments)
  uint16_t *dz_vals;      // [M][T][E] out
  uint16_t *dz_ovf;       // [cap][tw] out (rows at the forward's backup ranks)
};

template <int TW>
__global__ void __launch_bounds__(kSdThreads, 1)
    k_sddmm(const __grid_constant__ CUtensorMap tmap_dy, const __grid_constant__ CUtensorMap tmap_wd,
            const SddParams P) {
  constexpr int TILES_PER_ACC = kSdN / TW;
  constexpr int SP = TW + 1;                            // scratch row pitch (odd: no bank conflicts)
  constexpr uint32_t IDESC = idesc_bf16_f32(kBlockM, kSdN, 0, 0);
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t *smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  uint8_t *sA = smem;
  uint8_t *sB = smem + kSdStages * kSdABytes;
  float *scr = reinterpret_cast<float *>(sB + kSdStages * kSdBBytes);   // [128][SP]
  uint64_t *bars = reinterpret_cast<uint64_t *>(scr + kBlockM * SP + 2);
  uint64_t *full = bars;
  uint64_t *empty = bars + kSdStages;
  uint64_t *tm_full = bars + 2 * kSdStages;
  uint64_t *tm_empty = tm_full + 2;
  uint64_t *drain = tm_full + 4;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tm_full + 5);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const TwellView &H = P.h;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kSdStages; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
    for (int i = 0; i < 2; ++i) { mbar_init(&tm_full[i], 1); mbar_init(&tm_empty[i], 4); }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmap_dy);
    tma_prefetch_desc(&tmap_wd);
  }
  if (warp == 1) { tmem_alloc(tmem_slot, 512); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int num_tiles = P.num_m_blocks * P.num_n_blocks;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0; uint32_t phase = 0; uint32_t filled = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        const int m_blk = tile % P.num_m_blocks, n_blk = tile / P.num_m_blocks;
        for (int kb = 0; kb < P.num_kb; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) { ok = false; break; }
          mbar_arrive_expect_tx(&full[stage], kSdABytes + kSdBBytes);
          filled |= 1u << stage;
          tma_load_2d(sA + stage * kSdABytes, &tmap_dy, &full[stage], kb * kBlockK, m_blk * kBlockM);
          tma_load_2d(sB + stage * kSdBBytes, &tmap_wd, &full[stage], kb * kBlockK, n_blk * kSdN);
          if (++stage == kSdStages) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) {
        *abort_flag = 1;
        raise_status(H.status, TWELL_ERR_TIMEOUT);
        for (int i = 0; i < kSdStages; ++i) {
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
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++it) {
        const int acc = it & 1;
        if (!mbar_wait(&tm_empty[acc], (static_cast<uint32_t>(it >> 1) & 1u) ^ 1u, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kSdN);
        for (int kb = 0; kb < P.num_kb; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + stage * kSdABytes);
          const uint32_t b_addr = smem_u32(sB + stage * kSdBBytes);
#pragma unroll
          for (int k = 0; k < kBlockK / kUmmaK; ++k)
            umma_bf16(d_tmem, smem_desc_sw128(a_addr + k * 32, 16, 1024),
                      smem_desc_sw128(b_addr + k * 32, 16, 1024), IDESC, (kb | k) != 0);
          umma_commit(&empty[stage]);
          if (++stage == kSdStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma_commit(&tm_full[acc]);
      }
      if (!ok) {
        *abort_flag = 1;
        raise_status(H.status, TWELL_ERR_TIMEOUT);
      }
      umma_commit(drain);
      mbar_wait_bounded(drain, 0);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // thread = token row: the row's dH values of a hidden tile go to its own
    // scratch row, then the forward's slots pick theirs (independent loads of
    // the slot indices); an overflowing pair writes its masked dense segment at
    // the forward's backup rank.
    const int q = warp & 3;
    const int row_in_tile = q * 32 + lane;
    float *srow = scr + row_in_tile * SP;
    const int E = H.E, Tn = H.T;
    const int n_ovf = min(*H.n_ovf, H.cap);
    int it = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++it) {
      const int m_blk = tile % P.num_m_blocks, n_blk = tile / P.num_m_blocks;
      const int acc = it & 1;
      if (!mbar_wait(&tm_full[acc], static_cast<uint32_t>(it >> 1) & 1u, abort_flag)) {
        *abort_flag = 1;
        raise_status(H.status, TWELL_ERR_TIMEOUT);
        break;
      }
      tc_fence_after();
      const int r = m_blk * kBlockM + row_in_tile;
      const bool valid = r < P.M;
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * kSdN);
#pragma unroll 1
      for (int u = 0; u < TILES_PER_ACC; ++u) {
        const int t = n_blk * TILES_PER_ACC + u;
#pragma unroll 1
        for (int c = 0; c < TW / 32; ++c) {
          uint32_t v[32];
          __syncwarp();
          tmem_ld_32x32b_x32(t_row + u * TW + c * 32, v);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) srow[c * 32 + j] = __uint_as_float(v[j]);
        }
        if (!valid || t >= Tn) continue;
        const size_t pair = static_cast<size_t>(r) * Tn + t;
        const int n = __ldg(H.nnz + pair);
        const int ns = min(n, E);
        const uint8_t *ip = H.idx + pair * E;
        uint16_t *dv = P.dz_vals + pair * E;
        if ((E & 7) == 0) {
          // eight slots at a time: one 8-byte load of their indices, one 16-byte
          // store of their values (padding slots included)
          for (int s0 = 0; s0 < E; s0 += 8) {
            const uint2 iq = __ldg(reinterpret_cast<const uint2 *>(ip + s0));
            uint32_t w[4];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const uint32_t j = ((i < 4 ? iq.x : iq.y) >> (8 * (i & 3))) & (TW - 1);   // (indices are < tile_w)
              const uint32_t b = bf16_bits_rn(srow[j]);
              const uint32_t v = (s0 + i < ns && (b & 0x7FFFu)) ? b : 0u;              // -0 stored as +0
              if (i & 1) w[i >> 1] |= v << 16; else w[i >> 1] = v;
            }
            *reinterpret_cast<uint4 *>(dv + s0) = make_uint4(w[0], w[1], w[2], w[3]);
          }
        } else {
          for (int s = 0; s < ns; ++s) {
            const uint32_t b = bf16_bits_rn(srow[__ldg(ip + s) & (TW - 1)]);   // (indices are < tile_w)
            dv[s] = static_cast<uint16_t>((b & 0x7FFFu) ? b : 0u);   // -0 stored as +0
          }
          for (int s = ns; s < E; ++s) dv[s] = 0;                    // padding slots
        }
        if (n > E) {
          const int k = ovf_lower_bound(H.ovf_pos, n_ovf, static_cast<int>(pair));
          if (k < n_ovf && __ldg(H.ovf_pos + k) == static_cast<int>(pair)) {
            const uint16_t *hs = H.ovf_dense + static_cast<size_t>(k) * TW;
            uint16_t *ds = P.dz_ovf + static_cast<size_t>(k) * TW;
            for (int j = 0; j < TW; j += 8) {
              const uint4 m = __ldg(reinterpret_cast<const uint4 *>(hs + j));
              const uint32_t mw[4] = {m.x, m.y, m.z, m.w};
              uint32_t o[4];
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                uint32_t lo = bf16_bits_rn(srow[j + 2 * i]), hi = bf16_bits_rn(srow[j + 2 * i + 1]);
                lo = ((mw[i] & 0x7FFFu) && (lo & 0x7FFFu)) ? lo : 0u;
                hi = ((mw[i] & 0x7FFF0000u) && (hi & 0x7FFFu)) ? hi : 0u;
                o[i] = lo | (hi << 16);
              }
              *reinterpret_cast<uint4 *>(ds + j) = make_uint4(o[0], o[1], o[2], o[3]);
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
    tmem_dealloc(tmem_base, 512);
  }
}

// ============================================================================ transpose
constexpr int kTrTok = 128;     // tokens per output tile (the transposed tile width)
constexpr int kTrUnits = 128;   // hidden units per CTA

struct TrParams {
  TwellView a;            // input [M x f], tiles over f
  PackTarget out;         // output [f x M], tiles of 128 tokens (out.M = f, out.f = M)
  float *sum_part;        // NULL, or [f][M / 128]: per (unit, token tile) sum of values
};

__global__ void __launch_bounds__(256) k_twell_transpose(const TrParams P) {
  // dynamic shared memory: the dense block D [128 tokens][128 units] bf16, then
  // per unit its output record (E values, E indices) before the vector stores
  extern __shared__ __align__(16) uint8_t tr_smem[];
  uint16_t (*D)[kTrUnits] = reinterpret_cast<uint16_t (*)[kTrUnits]>(tr_smem);
  griddep_wait();   // the input's writes (a dependent launch after its producer)
  const TwellView &A = P.a;
  const PackTarget &O = P.out;
  const int E = O.E, T = O.T;
  uint16_t *rec_v = reinterpret_cast<uint16_t *>(tr_smem + kTrTok * kTrUnits * 2);   // [128][E]
  uint8_t *rec_i = reinterpret_cast<uint8_t *>(rec_v + kTrUnits * E);                // [128][E]
  const int tau = blockIdx.y;                     // token tile
  const int u0 = blockIdx.x * kTrUnits;           // first hidden unit
  const int tid = threadIdx.x;
  for (int i = tid; i < kTrTok * kTrUnits / 8; i += blockDim.x)
    reinterpret_cast<uint4 *>(&D[0][0])[i] = make_uint4(0u, 0u, 0u, 0u);
  __syncthreads();
  // --- rows: token threads scatter their slots (or backup segments) of the
  //     hidden tiles covering units [u0, u0 + 128)
  const int tiles = kTrUnits / A.tw;              // tile_w <= 128
  const int n_ovf = min(*A.n_ovf, A.cap);
  for (int w = tid; w < kTrTok * tiles; w += blockDim.x) {
    const int rl = w % kTrTok, tl = w / kTrTok;
    const int r = tau * kTrTok + rl;
    const int t = u0 / A.tw + tl;
    if (r >= A.M || t >= A.T) continue;
    const size_t pair = static_cast<size_t>(r) * A.T + t;
    const int n = __ldg(A.nnz + pair);
    if (n == 0) continue;
    uint16_t *drow = &D[rl][tl * A.tw];
    if (n <= A.E) {
      for (int s = 0; s < n; ++s) {
        const int j = __ldg(A.idx + pair * A.E + s);
        if (j < A.tw) drow[j] = __ldg(A.vals + pair * A.E + s);
      }
    } else {
      const int k = ovf_lower_bound(A.ovf_pos, n_ovf, static_cast<int>(pair));
      if (k < n_ovf && __ldg(A.ovf_pos + k) == static_cast<int>(pair)) {
        const uint4 *src = reinterpret_cast<const uint4 *>(A.ovf_dense + static_cast<size_t>(k) * A.tw);
        for (int j = 0; j < A.tw / 8; ++j) reinterpret_cast<uint4 *>(drow)[j] = __ldg(src + j);
      }
    }
  }
  __syncthreads();
  // --- columns: unit threads pack their column in token order into shared
  //     memory, then store the record with 16-byte stores
  if (tid < kTrUnits) {
    const int u = u0 + tid;
    if (u < O.M) {
      const size_t pair = static_cast<size_t>(u) * T + tau;
      uint16_t *sv = rec_v + tid * E;
      uint8_t *si = rec_i + tid * E;
      int cnt = 0;
      float sum = 0.f;
      for (int r = 0; r < kTrTok; ++r) {
        const uint16_t hv = D[r][tid];
        if ((hv & 0x7FFFu) == 0) continue;
        sum += __uint_as_float(static_cast<uint32_t>(hv) << 16);
        if (cnt < E) { sv[cnt] = hv; si[cnt] = static_cast<uint8_t>(r); }
        ++cnt;
      }
      for (int s = cnt; s < E; ++s) { sv[s] = 0; si[s] = 0; }
      uint16_t *ov = O.vals + pair * E;
      uint8_t *oi = O.idx + pair * E;
      if ((E & 15) == 0) {            // records 16-byte aligned: vector stores
        for (int s = 0; s < E; s += 8) *reinterpret_cast<uint4 *>(ov + s) = *reinterpret_cast<const uint4 *>(sv + s);
        for (int s = 0; s < E; s += 16) *reinterpret_cast<uint4 *>(oi + s) = *reinterpret_cast<const uint4 *>(si + s);
      } else if ((E & 7) == 0) {
        for (int s = 0; s < E; s += 8) {
          *reinterpret_cast<uint4 *>(ov + s) = *reinterpret_cast<const uint4 *>(sv + s);
          *reinterpret_cast<uint2 *>(oi + s) = *reinterpret_cast<const uint2 *>(si + s);
        }
      } else {
        for (int s = 0; s < E; ++s) { ov[s] = sv[s]; oi[s] = si[s]; }
      }
      O.nnz[pair] = static_cast<uint16_t>(cnt);
      if (P.sum_part != nullptr) P.sum_part[pair] = sum;
      if (cnt > E) {   // stage the dense column segment for the backup ordering
        const int k = atomicAdd(O.stage_ctr, 1);
        atomicAdd(O.row_ovf + u, 1);
        if (k < O.cap) {
          O.stage_pos[k] = static_cast<int32_t>(pair);
          uint16_t *dst = O.stage_dense + static_cast<size_t>(k) * kTrTok;
          for (int r = 0; r < kTrTok; r += 8) {
            uint32_t w[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const uint32_t lo = D[r + 2 * i][tid], hi = D[r + 2 * i + 1][tid];
              w[i] = ((lo & 0x7FFFu) ? lo : 0u) | (((hi & 0x7FFFu) ? hi : 0u) << 16);
            }
            *reinterpret_cast<uint4 *>(dst + r) = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
      }
    }
  }
}

}  // namespace

cudaError_t launch_sddmm(const TwellView &h, const uint16_t *dy, const uint16_t *w_down, int d,
                         uint16_t *dz_vals, uint16_t *dz_ovf, int num_sms, cudaStream_t s) {
  if (h.M == 0) return cudaSuccess;
  if (h.tw > 128) return cudaErrorNotSupported;
  CUtensorMap mdy, mwd;
  if (encode_tensor_map_2d(&mdy, dy, d, h.M, static_cast<uint64_t>(d) * 2, kBlockK, kBlockM,
                           CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  if (encode_tensor_map_2d(&mwd, w_down, d, h.f, static_cast<uint64_t>(d) * 2, kBlockK, kSdN,
                           CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  SddParams P;
  P.M = h.M; P.d = d; P.f = h.f;
  P.num_m_blocks = (h.M + kBlockM - 1) / kBlockM;
  P.num_n_blocks = (h.f + kSdN - 1) / kSdN;
  P.num_kb = d / kBlockK;
  P.h = h;
  P.dz_vals = dz_vals;
  P.dz_ovf = dz_ovf;
  const size_t smem = 1024 + kSdStages * (kSdABytes + kSdBBytes) +
                      static_cast<size_t>(kBlockM) * (h.tw + 1) * 4 + 16 + 256;
  const int tiles = P.num_m_blocks * P.num_n_blocks;
  const dim3 grid(tiles < num_sms ? tiles : num_sms), block(kSdThreads);
  cudaError_t e;
  switch (h.tw) {
    case 32:
      e = cudaFuncSetAttribute(k_sddmm<32>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
      return e != cudaSuccess ? e : launch_k(k_sddmm<32>, grid, block, smem, s, false, 1, mdy, mwd, P);
    case 64:
      e = cudaFuncSetAttribute(k_sddmm<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
      return e != cudaSuccess ? e : launch_k(k_sddmm<64>, grid, block, smem, s, false, 1, mdy, mwd, P);
    case 128:
      e = cudaFuncSetAttribute(k_sddmm<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
      return e != cudaSuccess ? e : launch_k(k_sddmm<128>, grid, block, smem, s, false, 1, mdy, mwd, P);
    default:
      return cudaErrorNotSupported;
  }
}

cudaError_t launch_twell_transpose(const TwellView &a, const PackTarget &out, float *sum_part, bool pdl,
                                   cudaStream_t s) {
  if (a.M == 0) return cudaSuccess;
  if (a.tw > kTrUnits || out.tw != kTrTok || a.M % kTrTok != 0 || a.f % kTrUnits != 0)
    return cudaErrorNotSupported;
  TrParams P;
  P.a = a;
  P.out = out;
  P.sum_part = sum_part;
  const dim3 grid(a.f / kTrUnits, a.M / kTrTok), block(256);
  // D, then the staged records (E values and E indices per unit, 16-byte aligned)
  const size_t smem = static_cast<size_t>(kTrTok) * kTrUnits * 2 +
                      ((static_cast<size_t>(kTrUnits) * out.E * 3 + 15) & ~static_cast<size_t>(15));
  cudaError_t e = cudaFuncSetAttribute(k_twell_transpose, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  return launch_k(k_twell_transpose, grid, block, smem, s, pdl, 1, P);
}

}  // namespace twell
