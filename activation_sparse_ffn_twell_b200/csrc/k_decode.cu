// Decode-size batches (M <= 256 tokens): both projections with the tokens on
// the MMA's N side, so that every SM streams its own slice of the weights.
//
// At a few hundred tokens the layer is bound by reading W_up and W_down from
// HBM, and the 128-token tiles of the main kernels cover only a few SMs.  Here:
//
//   k_up_pack_dec   one CTA per 128 hidden units: D[unit][token] = W_up x^T
//                   (M = 128 units, N = tokens, K = d_model).  The whole token
//                   batch sits in one accumulator; the epilogue (thread = hidden
//                   unit, TMEM lane) applies bias + ReLU (x up when gated),
//                   rounds to bf16 and packs each (token, tile) pair's nonzeros
//                   into its TwELL slots with warp ballots plus a cross-warp
//                   prefix -- the same TwELL rule as the token-major producer
//                   (upppp.jp 2026-05-11, section
//                   「TwELLとカスタムCUDAカーネルが解決する課題」), including the
//                   dense backup of pairs with more than ell_w nonzeros.
//
//   k_spmm_dec      y^T = W_down^T h^T, split-K over a thread-block cluster:
//                   a cluster owns 128 output columns, each of its CTAs a range
//                   of hidden K steps.  The W_down tile [64 hidden x 128 cols]
//                   is an M-major A operand loaded by TMA; the h^T operand
//                   [tokens x 64 hidden] is rebuilt in shared memory from the
//                   TwELL slots (and backup segments) by builder warps.  The
//                   fp32 partial sums meet in the CTAs' shared memory and are
//                   added through distributed shared memory, in a fixed order,
//                   before the one bf16 rounding of y.
#include <cstdlib>

#include "twell_device.cuh"

namespace twell {
namespace {

constexpr int kDecUnits = 128;                           // hidden units (MMA M) per up CTA
constexpr int kDecCols = 128;                            // y columns (MMA M) per down cluster
constexpr int kDecMaxStages = 12;
constexpr int kDecMaxTokens = 256;
constexpr int kWBytes = kDecUnits * kBlockK * 2;         // 16 KB weight tile per K step
constexpr int kDecEpiGroups = 3;                         // up epilogue: groups of 4 warps
constexpr int kDecUpThreads = 64 + kDecEpiGroups * 128;   // TMA, MMA, epilogue warps
constexpr int kDecDownThreads = 448;                     // TMA, MMA, 4 epilogue, 8 builder warps
constexpr size_t kDecSmemBudget = 225 * 1024;
// K steps per pipeline stage of the up kernel: two adjacent 64-column boxes of
// each weight row per stage, so the rows are read in 256-byte pieces (one K step
// per stage when gated: W_up and W_gate tiles already fill a stage).
template <bool GATED> constexpr int dec_up_kps() { return GATED ? 1 : 2; }

uint32_t tmem_cols_for(int cols) {
  uint32_t c = 32;
  while (c < static_cast<uint32_t>(cols)) c <<= 1;
  return c;
}

// ============================================================================ up + pack
struct DecUpParams {
  const uint16_t *b;
  int M, d, f;
  int np;                 // MMA N: tokens rounded up to a multiple of 16
  int acc_up;             // TMEM column of the up-branch accumulator (gated)
  int num_kb, num_ub, stages;
  uint32_t tmem_cols, idesc;
  float *z_debug;
  float *l1_part;         // NULL, or [M][T]: per (token, tile) sum of |h|
  PackTarget out;
};

template <int TW, bool GATED>
__global__ void __launch_bounds__(kDecUpThreads, 1)
    k_up_pack_dec(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                  const __grid_constant__ CUtensorMap tmap_g, const DecUpParams P) {
  constexpr int WPT = TW / 32;                            // epilogue warps per hidden tile
  constexpr int W_BYTES = (GATED ? 2 : 1) * kWBytes;     // [W_up tile][W_gate tile]
  griddep_launch_dependents();   // the backup scan waits for this grid anyway
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t *smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  const int kStages = P.stages;
  constexpr int KPS = dec_up_kps<GATED>();
  const int XB = P.np * 128;                              // x tile of one K step
  const int STAGE = KPS * (W_BYTES + XB);                 // [KPS weight tiles][KPS x tiles]
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kStages * STAGE);
  uint64_t *full = bars;
  uint64_t *empty = bars + kDecMaxStages;
  uint64_t *tm_full = bars + 2 * kDecMaxStages;
  uint64_t *tm_empty = tm_full + 1;
  uint64_t *drain = tm_full + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tm_full + 3);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  int *cnt_all = reinterpret_cast<int *>(tm_full + 4);    // [group][4 warps][32 tokens]
  int *ovk_all = cnt_all + kDecEpiGroups * 128;           // [group][tiles in CTA][32 tokens]
  float *l1_all = reinterpret_cast<float *>(ovk_all + kDecEpiGroups * 128);   // [group][4 warps][32]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const PackTarget &O = P.out;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
    mbar_init(tm_full, 1);
    mbar_init(tm_empty, 4 * kDecEpiGroups);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmap_x);
    tma_prefetch_desc(&tmap_w);
    if (GATED) tma_prefetch_desc(&tmap_g);
  }
  if (warp == 1) { tmem_alloc(tmem_slot, P.tmem_cols); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0; uint32_t phase = 0;
      uint32_t filled = 0;
      bool ok = true;
      for (int ub = blockIdx.x; ub < P.num_ub && ok; ub += gridDim.x) {
        for (int kb0 = 0; kb0 < P.num_kb; kb0 += KPS) {
          const int nk = min(KPS, P.num_kb - kb0);
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) { ok = false; break; }
          // the x box is M rows; operand rows M..np-1 feed accumulator columns
          // that no one reads
          mbar_arrive_expect_tx(&full[stage], static_cast<uint32_t>(nk * (W_BYTES + P.M * 128)));
          filled |= 1u << stage;
          uint8_t *dst = smem + stage * STAGE;
          for (int j = 0; j < nk; ++j) {
            const int kb = kb0 + j;
            tma_load_2d(dst + j * W_BYTES, &tmap_w, &full[stage], kb * kBlockK, ub * kDecUnits);
            if constexpr (GATED)
              tma_load_2d(dst + j * W_BYTES + kWBytes, &tmap_g, &full[stage], kb * kBlockK, ub * kDecUnits);
            tma_load_2d(dst + KPS * W_BYTES + j * XB, &tmap_x, &full[stage], kb * kBlockK, 0);
          }
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) {
        *abort_flag = 1;
        raise_status(O.status, TWELL_ERR_TIMEOUT);
        for (int i = 0; i < kStages; ++i) {   // let issued copies land
          if (!((filled >> i) & 1u)) continue;
          mbar_wait_bounded(&full[i], (i < stage) ? phase : (phase ^ 1u));
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0; uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      for (int ub = blockIdx.x; ub < P.num_ub && ok; ub += gridDim.x, ++it) {
        if (!mbar_wait(tm_empty, static_cast<uint32_t>(it & 1) ^ 1u, abort_flag)) { ok = false; break; }
        tc_fence_after();
        for (int kb0 = 0; kb0 < P.num_kb; kb0 += KPS) {
          const int nk = min(KPS, P.num_kb - kb0);
          if (!mbar_wait(&full[stage], phase, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t s_addr = smem_u32(smem + stage * STAGE);
          for (int j = 0; j < nk; ++j) {
            const uint32_t w_addr = s_addr + j * W_BYTES;
            const uint32_t x_addr = s_addr + KPS * W_BYTES + j * XB;
#pragma unroll
            for (int k = 0; k < kBlockK / kUmmaK; ++k) {
              const uint64_t xdesc = smem_desc_sw128(x_addr + k * 32, 16, 1024);
              const uint32_t acc = ((kb0 + j) | k) != 0;
              if constexpr (GATED) {
                umma_bf16(tmem_base, smem_desc_sw128(w_addr + kWBytes + k * 32, 16, 1024), xdesc, P.idesc, acc);
                umma_bf16(tmem_base + P.acc_up, smem_desc_sw128(w_addr + k * 32, 16, 1024), xdesc, P.idesc, acc);
              } else {
                umma_bf16(tmem_base, smem_desc_sw128(w_addr + k * 32, 16, 1024), xdesc, P.idesc, acc);
              }
            }
          }
          umma_commit(&empty[stage]);
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma_commit(tm_full);
      }
      if (!ok) {
        *abort_flag = 1;
        raise_status(O.status, TWELL_ERR_TIMEOUT);
      }
      umma_commit(drain);
      mbar_wait_bounded(drain, 0);
    }
  } else {
    // ------------------------------------------------------------ epilogue + pack
    griddep_wait();   // the call's reset kernel (counters, status) precedes the writes
    // thread = hidden unit (TMEM lane); a hidden tile spans WPT warps, whose
    // nonzero counts are combined through shared memory per 32-token chunk.
    // kDecEpiGroups groups of 4 warps (one per TMEM lane quarter) take the
    // 32-token chunks in turn, each group with its own named barrier.
    const int grp = (warp - 2) >> 2;
    int *cnt_s = cnt_all + grp * 128;
    int *ovk_s = ovk_all + grp * 128;
    float *l1_s = l1_all + grp * 128;
    const uint32_t bar_id = 1u + static_cast<uint32_t>(grp);
    const int q = warp & 3;                  // TMEM lane quarter
    const int li = q % WPT;                  // this warp's place inside its hidden tile
    const int tl = q / WPT;                  // the tile's place inside the CTA's 128 units
    const int in_tile = 32 * li + lane;
    const unsigned lt = (1u << lane) - 1u;
    const int E = O.E, T = O.T;
    const uint32_t trow = tmem_base + (static_cast<uint32_t>(32 * q) << 16);
    // Every epilogue warp runs the same sequence of named barriers whatever
    // happens: after a failed wait it keeps stepping through them with no work.
    bool ok = true;
    int it = 0;
    for (int ub = blockIdx.x; ub < P.num_ub; ub += gridDim.x, ++it) {
      if (ok && !mbar_wait(tm_full, static_cast<uint32_t>(it & 1), abort_flag)) {
        ok = false;
        *abort_flag = 1;
        raise_status(O.status, TWELL_ERR_TIMEOUT);
      }
      tc_fence_after();
      const int unit = ub * kDecUnits + 32 * q + lane;
      const int t = (ub * kDecUnits + 32 * q) / TW;
      const float bias = (P.b != nullptr) ? __uint_as_float(static_cast<uint32_t>(__ldg(P.b + unit)) << 16) : 0.f;
      const int nchunks = (P.M + 31) >> 5;
#pragma unroll 1
      for (int c0 = grp; c0 < nchunks; c0 += kDecEpiGroups) {
        // pass 1: h, and this warp's nonzero count per token (lane j keeps token j's)
        uint32_t hb[32];
        int myc = 0;
        if (ok) {
          uint32_t a[32];
          uint32_t g[GATED ? 32 : 1];
          __syncwarp();
          tmem_ld_32x32b_x32(trow + c0 * 32, a);
          if constexpr (GATED) tmem_ld_32x32b_x32(trow + P.acc_up + c0 * 32, g);
          tmem_ld_wait();
          if (P.z_debug != nullptr) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const int r = c0 * 32 + j;
              if (r >= P.M) continue;
              float *zr = P.z_debug + static_cast<size_t>(r) * (GATED ? 2 * P.f : P.f);
              zr[unit] = __uint_as_float(a[j]);
              if constexpr (GATED) zr[P.f + unit] = __uint_as_float(g[j]);
            }
          }
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            // separately rounded fp32 add / multiply (no contraction), one bf16 rounding
            float v = fmaxf(__fadd_rn(__uint_as_float(a[j]), bias), 0.f);
            if constexpr (GATED) v = __fmul_rn(v, __uint_as_float(g[j]));
            const uint32_t h = bf16_bits_rn(v);
            hb[j] = (h & 0x7FFFu) ? h : 0u;    // -0 is stored as +0
            const unsigned m = __ballot_sync(0xFFFFFFFFu, hb[j] != 0u);
            if (lane == j) myc = __popc(m);
          }
        }
        cnt_s[q * 32 + lane] = myc;
        if (P.l1_part != nullptr) {
          // this warp's sum of |h| per token: a transposed butterfly leaves the
          // sum for token `lane` of the chunk in lane `lane` (fixed order)
          float v[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = ok ? fabsf(__uint_as_float(hb[j] << 16)) : 0.f;
#pragma unroll
          for (int sh = 16; sh >= 1; sh >>= 1) {
            const bool upper = (lane & sh) != 0;
#pragma unroll
            for (int i = 0; i < sh; ++i) {
              const float send = upper ? v[i] : v[i + sh];
              const float keep = upper ? v[i + sh] : v[i];
              v[i] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, sh);
            }
          }
          l1_s[q * 32 + lane] = v[0];
        }
        named_bar_sync(bar_id, 128);
        // pass 2: per token (lane = token of the chunk) the tile total and the
        // nonzeros of the tile's lower warps; the tile's first warp writes nnz
        // and claims a staging slot for an overflowing pair
        const int rl = c0 * 32 + lane;
        int base_l = 0, tot_l = 0;
#pragma unroll
        for (int w = 0; w < WPT; ++w) {
          const int c = cnt_s[(q - li + w) * 32 + lane];
          tot_l += c;
          if (w < li) base_l += c;
        }
        if (li == 0) {
          int k = -1;
          if (ok && rl < P.M) {
            const size_t pair = static_cast<size_t>(rl) * T + t;
            O.nnz[pair] = static_cast<uint16_t>(tot_l);
            if (P.l1_part != nullptr) {   // the tile's warps in order
              float l1t = 0.f;
              for (int w = 0; w < WPT; ++w) l1t += l1_s[(q + w) * 32 + lane];
              P.l1_part[pair] = l1t;
            }
            if (tot_l > E) {
              k = atomicAdd(O.stage_ctr, 1);
              atomicAdd(O.row_ovf + rl, 1);
              if (k < O.cap) O.stage_pos[k] = static_cast<int32_t>(pair);
            }
          }
          ovk_s[tl * 32 + lane] = k;
        }
        named_bar_sync(bar_id, 128);
        if (!ok) continue;
        // pass 3: slots, padding, dense backup segment
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int r = c0 * 32 + j;
          if (r >= P.M) continue;   // same for the whole warp
          const int tot = __shfl_sync(0xFFFFFFFFu, tot_l, j);
          const int base = __shfl_sync(0xFFFFFFFFu, base_l, j);
          const bool nz = hb[j] != 0u;
          const unsigned m = __ballot_sync(0xFFFFFFFFu, nz);
          const size_t rec = (static_cast<size_t>(r) * T + t) * E;
          if (nz) {
            const int s = base + __popc(m & lt);
            if (s < E) {
              O.vals[rec + s] = static_cast<uint16_t>(hb[j]);
              O.idx[rec + s] = static_cast<uint8_t>(in_tile);
            }
          }
          if (li == WPT - 1) {
            for (int s = tot + lane; s < E; s += 32) { O.vals[rec + s] = 0; O.idx[rec + s] = 0; }
          }
          if (tot > E) {
            const int k = ovk_s[tl * 32 + j];
            if (k >= 0 && k < O.cap)
              O.stage_dense[static_cast<size_t>(k) * TW + in_tile] = static_cast<uint16_t>(hb[j]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tm_empty);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem_base, P.tmem_cols);
  }
}

// ============================================================================ down
struct DecDownParams {
  TwellView A;
  uint16_t *y;
  int d;
  int np;                 // MMA N: tokens rounded up to a multiple of 16
  int num_kb;             // hidden K steps of 64
  int split;              // CTAs per cluster (K ranges per 128 output columns)
  int stages;
  uint32_t tmem_cols, idesc;
};

// Clear one 128-byte operand row: each lane starts at a different 16-byte
// chunk, so the 32 rows of a warp spread over all banks.
__device__ __forceinline__ void zero_row_128(uint8_t *rp, int row) {
#pragma unroll
  for (int c = 0; c < 8; ++c)
    *reinterpret_cast<uint4 *>(rp + (((c + row) & 7) << 4)) = make_uint4(0u, 0u, 0u, 0u);
}

// EV: ell_w / 8 on the fast builder path (ell_w % 8 == 0, tile_w >= 64), else 0.
template <int EV>
__global__ void __launch_bounds__(kDecDownThreads, 1)
    k_spmm_dec(const __grid_constant__ CUtensorMap tmap_wd, const DecDownParams P) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t *smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  const int kStages = P.stages;
  const int STAGE = kWBytes + P.np * 128;                 // [W_down tile][h^T tile]
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kStages * STAGE);
  uint64_t *full = bars;
  uint64_t *empty = bars + kDecMaxStages;
  uint64_t *tm_full = bars + 2 * kDecMaxStages;
  uint64_t *drain = tm_full + 1;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tm_full + 2);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  // after the K loop the stage buffers hold this CTA's fp32 partial [np][128]
  float *part = reinterpret_cast<float *>(smem);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const TwellView &A = P.A;
  const uint32_t rank = cluster_ctarank();
  const int col0 = static_cast<int>(cluster_id_x()) * kDecCols;     // first y column
  const int kb_lo = static_cast<int>((static_cast<long long>(rank) * P.num_kb) / P.split);
  const int kb_hi = static_cast<int>((static_cast<long long>(rank + 1) * P.num_kb) / P.split);

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) { mbar_init(&full[i], 1 + 8); mbar_init(&empty[i], 1); }
    mbar_init(tm_full, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmap_wd);
  }
  if (warp == 1) { tmem_alloc(tmem_slot, P.tmem_cols); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // The W_down stream (warp 0) depends on no earlier kernel; every other role
  // reads TwELL or writes y, so it waits for the previous kernels of a
  // dependent launch here.
  if (warp != 0) griddep_wait();

  if (warp == 0) {
    // ------------------------------------------------------------ TMA: W_down tiles
    if (lane == 0) {
      int stage = 0; uint32_t phase = 0;
      uint32_t filled = 0;
      bool ok = true;
      for (int kb = kb_lo; kb < kb_hi; ++kb) {
        if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) { ok = false; break; }
        mbar_arrive_expect_tx(&full[stage], kWBytes);
        filled |= 1u << stage;
        uint8_t *dst = smem + stage * STAGE;
        // two 64-column boxes: an M-major operand, 64-element groups 8 KB apart
        // (columns past d_model are outside the tensor and arrive as zeros)
        tma_load_2d(dst, &tmap_wd, &full[stage], col0, kb * kBlockK);
        tma_load_2d(dst + 8192, &tmap_wd, &full[stage], col0 + 64, kb * kBlockK);
        if (++stage == kStages) { stage = 0; phase ^= 1u; }
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
      int stage = 0; uint32_t phase = 0;
      bool ok = true;
      for (int kb = kb_lo; kb < kb_hi; ++kb) {
        if (!mbar_wait(&full[stage], phase, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t w_addr = smem_u32(smem + stage * STAGE);
        const uint32_t h_addr = w_addr + kWBytes;
#pragma unroll
        for (int k = 0; k < kBlockK / kUmmaK; ++k) {
          // A (W_down^T): 16 hidden rows of 128 B per step; B (h^T): K-major rows
          const uint64_t adesc = smem_desc_sw128(w_addr + k * 2048, 8192, 1024);
          const uint64_t bdesc = smem_desc_sw128(h_addr + k * 32, 16, 1024);
          umma_bf16(tmem_base, adesc, bdesc, P.idesc, (kb != kb_lo || k != 0) ? 1u : 0u);
        }
        umma_commit(&empty[stage]);
        if (++stage == kStages) { stage = 0; phase ^= 1u; }
      }
      if (!ok) {
        *abort_flag = 1;
        raise_status(A.status, TWELL_ERR_TIMEOUT);
      }
      umma_commit(tm_full);   // also issued on abort: the epilogue must not wait out its limit
      umma_commit(drain);
      mbar_wait_bounded(drain, 0);
    }
  } else if (warp < 6) {
    // ------------------------------------------------------------ epilogue: TMEM -> partial
    const int q = warp & 3;
    if (mbar_wait(tm_full, 0, abort_flag)) {
      tc_fence_after();
      const uint32_t trow = tmem_base + (static_cast<uint32_t>(32 * q) << 16);
      const int c_local = 32 * q + lane;
      const int nchunks = (A.M + 31) >> 5;
      for (int c0 = 0; c0 < nchunks; ++c0) {
        uint32_t v[32];
        __syncwarp();
        tmem_ld_32x32b_x32(trow + c0 * 32, v);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int tok = c0 * 32 + j;
          if (tok < A.M) part[tok * kDecCols + c_local] = __uint_as_float(v[j]);
        }
      }
    } else {
      *abort_flag = 1;
      raise_status(A.status, TWELL_ERR_TIMEOUT);
    }
  } else {
    // ------------------------------------------------------------ builders: h^T tiles
    // thread = token row of the operand; row i of a stage holds hidden columns
    // [64 kb, 64 kb + 64) of token i, 128-byte swizzled
    const int row = (warp - 6) * 32 + lane;
    const bool live = row < A.M;
    const int tw = A.tw, E = A.E, Tn = A.T;
    const int n_ovf = min(*A.n_ovf, A.cap);
    const uint32_t row_swz = static_cast<uint32_t>(row & 7);
    int stage = 0; uint32_t phase = 0;
    bool ok = true;
    if constexpr (EV > 0) {
      // tile_w >= 64: a K step lies inside one hidden tile.  The row's record
      // of the next tile (values, indices, count) is loaded into registers
      // while the current tile is written, so no K step waits on its loads.
      constexpr int EF = 8 * EV;
      const int lg_tw = 31 - __clz(tw);
      const size_t pair0 = static_cast<size_t>(live ? row : 0) * Tn;
      auto fetch = [&](int t, uint4 (&v)[EV], uint2 (&ix)[EV], int &n) {
        if (live && t < Tn) {
          const uint4 *gv = reinterpret_cast<const uint4 *>(A.vals + (pair0 + t) * EF);
          const uint2 *gi = reinterpret_cast<const uint2 *>(A.idx + (pair0 + t) * EF);
#pragma unroll
          for (int g = 0; g < EV; ++g) { v[g] = __ldg(gv + g); ix[g] = __ldg(gi + g); }
          n = static_cast<int>(__ldg(A.nnz + pair0 + t));
        } else {
          n = 0;
        }
      };
      uint4 vq[EV], vq1[EV];
      uint2 iq[EV], iq1[EV];
      int cur_t = -1, n0 = 0, n1 = 0, ovf_k = -1;
      // this row's backup entries from the CTA's first tile on, in tile order
      int walk = live ? ovf_lower_bound(A.ovf_pos, n_ovf,
                                        static_cast<int>(pair0) + ((kb_lo * kBlockK) >> lg_tw))
                      : n_ovf;
      for (int kb = kb_lo; kb < kb_hi; ++kb) {
        const int t = (kb * kBlockK) >> lg_tw;
        if (t != cur_t) {
          if (cur_t < 0) {
            fetch(t, vq, iq, n0);
          } else {
#pragma unroll
            for (int g = 0; g < EV; ++g) { vq[g] = vq1[g]; iq[g] = iq1[g]; }
            n0 = n1;
          }
          fetch(t + 1, vq1, iq1, n1);
          cur_t = t;
          ovf_k = -1;
          if (n0 > EF && walk < n_ovf && __ldg(A.ovf_pos + walk) == static_cast<int>(pair0) + t)
            ovf_k = walk++;
        }
        if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) { ok = false; break; }
        if (row < P.np) {
          uint8_t *rp = smem + stage * STAGE + kWBytes + row * 128;
          zero_row_128(rp, row);
          const int base = (t << lg_tw) - kb * kBlockK;   // K-step column of in-tile index 0
          if (n0 > 0 && n0 <= EF) {
#pragma unroll
            for (int g = 0; g < EV; ++g) {
              const uint32_t vw[4] = {vq[g].x, vq[g].y, vq[g].z, vq[g].w};
              const uint32_t iw[2] = {iq[g].x, iq[g].y};
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                const uint32_t col = static_cast<uint32_t>(base + static_cast<int>((iw[e >> 2] >> (8 * (e & 3))) & 0xFFu));
                if (8 * g + e < n0 && col < static_cast<uint32_t>(kBlockK)) {
                  *reinterpret_cast<uint16_t *>(rp + ((((col >> 3) ^ row_swz) << 4) + ((col & 7u) << 1))) =
                      static_cast<uint16_t>(vw[e >> 1] >> (16 * (e & 1)));
                }
              }
            }
          } else if (ovf_k >= 0) {                        // dense backup segment
            const uint16_t *src = A.ovf_dense + static_cast<size_t>(ovf_k) * tw - base;
#pragma unroll
            for (int c = 0; c < kBlockK; c += 8)
              *reinterpret_cast<uint4 *>(rp + ((((static_cast<uint32_t>(c) >> 3) ^ row_swz)) << 4)) =
                  __ldg(reinterpret_cast<const uint4 *>(src + c));
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&full[stage]);
        if (++stage == kStages) { stage = 0; phase ^= 1u; }
      }
    } else {
      // any ell_w / tile_w: per K step, the row's count and slots are read
      // from global memory for the (one or two) tiles the step covers
      for (int kb = kb_lo; kb < kb_hi; ++kb) {
        if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) { ok = false; break; }
        if (row < P.np) {
          uint8_t *rp = smem + stage * STAGE + kWBytes + row * 128;
          zero_row_128(rp, row);
          if (live) {
            const int c_lo = kb * kBlockK;
            const int t_hi = min((c_lo + kBlockK - 1) / tw, Tn - 1);   // d_ff may end inside the step
            for (int t = c_lo / tw; t <= t_hi; ++t) {
              const size_t pair = static_cast<size_t>(row) * Tn + t;
              const int n = __ldg(A.nnz + pair);
              if (n == 0) continue;
              const int base = t * tw - c_lo;                // K-step column of in-tile index 0
              if (n <= E) {
                const uint16_t *sv = A.vals + pair * E;
                const uint8_t *si = A.idx + pair * E;
                for (int s = 0; s < n; ++s) {
                  const int col = base + __ldg(si + s);
                  if (col >= 0 && col < kBlockK) {
                    const uint32_t c = static_cast<uint32_t>(col);
                    *reinterpret_cast<uint16_t *>(rp + ((((c >> 3) ^ row_swz) << 4) + ((c & 7u) << 1))) = __ldg(sv + s);
                  }
                }
              } else {
                const int k = ovf_lower_bound(A.ovf_pos, n_ovf, static_cast<int>(pair));
                if (k < n_ovf && __ldg(A.ovf_pos + k) == static_cast<int>(pair)) {
                  const uint16_t *src = A.ovf_dense + static_cast<size_t>(k) * tw;
                  const int lo = max(0, base), hi = min(kBlockK, base + tw);
                  for (int c = lo; c < hi; c += 8) {
                    const uint32_t cc = static_cast<uint32_t>(c);
                    *reinterpret_cast<uint4 *>(rp + (((cc >> 3) ^ row_swz) << 4)) =
                        __ldg(reinterpret_cast<const uint4 *>(src + (c - base)));
                  }
                }
              }
            }
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&full[stage]);
        if (++stage == kStages) { stage = 0; phase ^= 1u; }
      }
    }
    if (!ok) {
      *abort_flag = 1;
      raise_status(A.status, TWELL_ERR_TIMEOUT);
    }
  }

  // ---- cluster reduction: CTA `rank` adds the partials of its share of tokens
  __syncwarp();
  cluster_sync();
  {
    const int per = (A.M + P.split - 1) / P.split;
    const int tok0 = static_cast<int>(rank) * per;
    const int ntok = max(0, min(A.M, tok0 + per) - tok0);
    for (int i = threadIdx.x; i < ntok * (kDecCols / 4); i += blockDim.x) {
      const int tok = tok0 + i / (kDecCols / 4);
      const int c4 = (i % (kDecCols / 4)) * 4;
      const int gc = col0 + c4;
      if (gc >= P.d) continue;
      const float *src = part + tok * kDecCols + c4;
      float4 acc = ld_shared_cluster_f4(map_to_cta(src, 0));
      for (int r = 1; r < P.split; ++r) {
        const float4 v = ld_shared_cluster_f4(map_to_cta(src, static_cast<uint32_t>(r)));
        acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
      }
      *reinterpret_cast<uint2 *>(P.y + static_cast<size_t>(tok) * P.d + gc) =
          make_uint2(pack_bf16x2(acc.x, acc.y), pack_bf16x2(acc.z, acc.w));
    }
  }
  tc_fence_before();
  __syncwarp();
  cluster_sync();   // no CTA leaves while a peer still reads its partial
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem_base, P.tmem_cols);
  }
}

int round_tokens(int M) { return M <= 16 ? 16 : (M + 15) & ~15; }




template <int TW, bool GATED>
cudaError_t launch_up_dec_impl(const UpArgs &a, const PackTarget &t, int num_sms, cudaStream_t s) {
  DecUpParams P;
  P.b = a.b;
  P.M = a.M; P.d = a.d; P.f = a.f;
  P.np = round_tokens(a.M);
  const int acc_w = (P.np + 31) & ~31;                   // accumulator pitch in TMEM columns
  P.acc_up = GATED ? acc_w : 0;
  P.tmem_cols = tmem_cols_for(GATED ? 2 * acc_w : acc_w);
  P.idesc = idesc_bf16_f32(kDecUnits, P.np, 0, 0);
  P.num_kb = a.d / kBlockK;
  P.num_ub = a.f / kDecUnits;
  P.z_debug = a.z_debug;
  P.l1_part = a.l1_part;
  P.out = t;
  const size_t stage = static_cast<size_t>(dec_up_kps<GATED>()) *
                       ((GATED ? 2 : 1) * static_cast<size_t>(kWBytes) + static_cast<size_t>(P.np) * 128);
  const size_t extra = 1024 + 6144;                      // alignment slack, barriers, counts
  int stages = static_cast<int>((kDecSmemBudget - extra) / stage);
  if (stages > kDecMaxStages) stages = kDecMaxStages;
  if (stages < 2) return cudaErrorInvalidValue;
  P.stages = stages;
  const size_t smem = extra + stages * stage;

  CUtensorMap mx, mw, mg;
  if (encode_tensor_map_2d(&mx, a.x, a.d, a.M, static_cast<uint64_t>(a.d) * 2, kBlockK, a.M,
                           CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  if (encode_tensor_map_2d(&mw, a.w_up, a.d, a.f, static_cast<uint64_t>(a.d) * 2, kBlockK, kDecUnits,
                           CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  mg = mw;
  if (GATED && encode_tensor_map_2d(&mg, a.w_gate, a.d, a.f, static_cast<uint64_t>(a.d) * 2, kBlockK,
                                    kDecUnits, CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(k_up_pack_dec<TW, GATED>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int grid = P.num_ub < num_sms ? P.num_ub : num_sms;
  // a dependent launch after the call's reset kernel (see the epilogue's wait)
  return launch_k(k_up_pack_dec<TW, GATED>, dim3(grid), dim3(kDecUpThreads), smem, s, true, 1, mx, mw, mg, P);
}

// Largest number of co-resident clusters of `split` CTAs of the down kernel
// (0 if that cluster shape cannot be scheduled at this shared-memory size).
int max_dec_clusters(int split, size_t smem) {
  static int cache[9] = {-1, -1, -1, -1, -1, -1, -1, -1, -1};
  if (cache[split] >= 0) return cache[split];
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(split, 1, 1);
  cfg.blockDim = dim3(kDecDownThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = split;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  // every instance of the kernel has the same block and shared-memory shape
  if (cudaOccupancyMaxActiveClusters(&n, k_spmm_dec<0>, &cfg) != cudaSuccess) {
    (void)cudaGetLastError();
    n = 0;
  }
  cache[split] = n;
  return n;
}

bool decode_enabled() {
  static int v = -1;
  if (v < 0) {
    const char *e = getenv("TWELL_DECODE_PATH");
    v = (e != nullptr && e[0] == '0') ? 0 : 1;
  }
  return v == 1;
}

}  // namespace

bool decode_up_eligible(int M, int d_ff, int tile_w) {
  return decode_enabled() && M > 0 && M <= kDecMaxTokens && tile_w <= kDecUnits && d_ff % kDecUnits == 0;
}

bool decode_down_eligible(int M) { return decode_enabled() && M > 0 && M <= kDecMaxTokens; }

cudaError_t launch_up_pack_decode(const UpArgs &a, const PackTarget &t, int num_sms, cudaStream_t s) {
  if (a.M == 0) return cudaSuccess;
  const bool gated = a.w_gate != nullptr;
  switch (t.tw) {
    case 32: return gated ? launch_up_dec_impl<32, true>(a, t, num_sms, s) : launch_up_dec_impl<32, false>(a, t, num_sms, s);
    case 64: return gated ? launch_up_dec_impl<64, true>(a, t, num_sms, s) : launch_up_dec_impl<64, false>(a, t, num_sms, s);
    case 128: return gated ? launch_up_dec_impl<128, true>(a, t, num_sms, s) : launch_up_dec_impl<128, false>(a, t, num_sms, s);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_spmm_decode(const TwellView &v, const uint16_t *w_down, int d, uint16_t *y, int num_sms,
                               bool pdl, cudaStream_t s) {
  if (v.M == 0) return cudaSuccess;
  DecDownParams P;
  P.A = v;
  P.y = y;
  P.d = d;
  P.np = round_tokens(v.M);
  P.num_kb = (v.f + kBlockK - 1) / kBlockK;
  P.tmem_cols = tmem_cols_for(P.np);
  P.idesc = idesc_bf16_f32(kDecCols, P.np, 1, 0);
  const size_t stage = static_cast<size_t>(kWBytes) + static_cast<size_t>(P.np) * 128;
  const size_t extra = 1024 + 512;
  int stages = static_cast<int>((kDecSmemBudget - extra) / stage);
  if (stages > kDecMaxStages) stages = kDecMaxStages;
  // the partial [np][128] fp32 reuses the stage buffers
  if (stages < 2 || static_cast<size_t>(stages) * stage < static_cast<size_t>(P.np) * kDecCols * 4)
    return cudaErrorInvalidValue;
  P.stages = stages;
  const size_t smem = extra + stages * stage;
  const int ev = (v.E % 8 == 0 && v.E <= 64 && v.tw >= 64) ? v.E / 8 : 0;
  void (*kern)(const CUtensorMap, const DecDownParams) = nullptr;
  switch (ev) {
    case 1: kern = k_spmm_dec<1>; break;
    case 2: kern = k_spmm_dec<2>; break;
    case 3: kern = k_spmm_dec<3>; break;
    case 4: kern = k_spmm_dec<4>; break;
    case 5: kern = k_spmm_dec<5>; break;
    case 6: kern = k_spmm_dec<6>; break;
    case 7: kern = k_spmm_dec<7>; break;
    case 8: kern = k_spmm_dec<8>; break;
    default: kern = k_spmm_dec<0>; break;
  }
  // the attribute is the full budget, so the occupancy query below sees the
  // same limit at every token count
  cudaError_t e = cudaFuncSetAttribute(k_spmm_dec<0>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kDecSmemBudget));
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(kDecSmemBudget));
  if (e != cudaSuccess) return e;
  // Split K so that the clusters fill the GPU: the cost of a split is the
  // number of waves of clusters times the K steps per CTA.
  const int n_slices = (d + kDecCols - 1) / kDecCols;
  int best = 1;
  long long best_cost = -1;
  for (int split = 1; split <= 8; split *= 2) {
    if (split > P.num_kb || (split > 1 && n_slices * split > 2 * num_sms)) break;
    const int mc = max_dec_clusters(split, kDecSmemBudget);
    if (mc <= 0) continue;
    const long long waves = (n_slices + mc - 1) / mc;
    const long long cost = waves * ((P.num_kb + split - 1) / split);
    if (best_cost < 0 || cost < best_cost) { best_cost = cost; best = split; }
  }
  P.split = best;
  CUtensorMap mw;
  if (encode_tensor_map_2d(&mw, w_down, d, v.f, static_cast<uint64_t>(d) * 2, 64, kBlockK,
                           CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  return launch_k(kern, dim3(n_slices * best), dim3(kDecDownThreads), smem, s, pdl,
                  static_cast<unsigned>(best), mw, P);
}

}  // namespace twell
