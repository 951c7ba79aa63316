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
  const uint16_t *w_down;   // [d_ff][d] (row gathers of the touched-unit kernel)
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

// ---- roles shared by the two split-K down kernels

// W_down tiles by TMA (one thread): K steps [kb_lo, kb_hi), two 64-column boxes
// per step (an M-major operand, 64-element groups 8 KB apart; columns past
// d_model are outside the tensor and arrive as zeros).
__device__ __forceinline__ void dec_down_tma(uint8_t *smem, int STAGE, int kStages, uint64_t *full,
                                             uint64_t *empty, volatile int *abort_flag, const CUtensorMap *tmap_wd,
                                             int col0, int kb_lo, int kb_hi, int32_t *status) {
  int stage = 0; uint32_t phase = 0;
  uint32_t filled = 0;
  bool ok = true;
  for (int kb = kb_lo; kb < kb_hi; ++kb) {
    if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) { ok = false; break; }
    mbar_arrive_expect_tx(&full[stage], kWBytes);
    filled |= 1u << stage;
    uint8_t *dst = smem + stage * STAGE;
    tma_load_2d(dst, tmap_wd, &full[stage], col0, kb * kBlockK);
    tma_load_2d(dst + 8192, tmap_wd, &full[stage], col0 + 64, kb * kBlockK);
    if (++stage == kStages) { stage = 0; phase ^= 1u; }
  }
  if (!ok) {
    *abort_flag = 1;
    raise_status(status, TWELL_ERR_TIMEOUT);
    for (int i = 0; i < kStages; ++i) {   // let issued copies land
      if (!((filled >> i) & 1u)) continue;
      mbar_wait_bounded(&full[i], (i < stage) ? phase : (phase ^ 1u));
    }
  }
}

// MMA issuer (one thread): n_steps K steps of the stage ring, A = W_down^T tile
// (M-major: 16 hidden rows of 128 B per MMA, the two 64-column halves 8 KB
// apart), B = h^T tile (K-major rows).  tm_full is committed also on abort, so
// the epilogue never waits out its limit.
__device__ __forceinline__ void dec_down_mma(uint8_t *smem, int STAGE, int kStages, uint64_t *full,
                                             uint64_t *empty, uint64_t *tm_full, uint64_t *drain,
                                             volatile int *abort_flag, uint32_t tmem_base, uint32_t idesc,
                                             int n_steps, int32_t *status) {
  int stage = 0; uint32_t phase = 0;
  bool ok = true;
  for (int i = 0; i < n_steps; ++i) {
    if (!mbar_wait(&full[stage], phase, abort_flag)) { ok = false; break; }
    tc_fence_after();
    const uint32_t w_addr = smem_u32(smem + stage * STAGE);
    const uint32_t h_addr = w_addr + kWBytes;
#pragma unroll
    for (int k = 0; k < kBlockK / kUmmaK; ++k) {
      const uint64_t adesc = smem_desc_sw128(w_addr + k * 2048, 8192, 1024);
      const uint64_t bdesc = smem_desc_sw128(h_addr + k * 32, 16, 1024);
      umma_bf16(tmem_base, adesc, bdesc, idesc, (i != 0 || k != 0) ? 1u : 0u);
    }
    umma_commit(&empty[stage]);
    if (++stage == kStages) { stage = 0; phase ^= 1u; }
  }
  if (!ok) {
    *abort_flag = 1;
    raise_status(status, TWELL_ERR_TIMEOUT);
  }
  umma_commit(tm_full);
  umma_commit(drain);
  mbar_wait_bounded(drain, 0);
}

// Epilogue warps 2..5 (TMEM lane quarter = warp % 4): the CTA's fp32 partial
// [M][128] into shared memory; zeros when the CTA had no K step.
__device__ __forceinline__ void dec_down_partial(float *part, uint64_t *tm_full, volatile int *abort_flag,
                                                 uint32_t tmem_base, int warp, int lane, int M, bool has_k,
                                                 int32_t *status) {
  const int q = warp & 3;
  if (mbar_wait(tm_full, 0, abort_flag)) {
    tc_fence_after();
    const uint32_t trow = tmem_base + (static_cast<uint32_t>(32 * q) << 16);
    const int c_local = 32 * q + lane;
    const int nchunks = (M + 31) >> 5;
    for (int c0 = 0; c0 < nchunks; ++c0) {
      uint32_t v[32];
      if (has_k) {
        __syncwarp();
        tmem_ld_32x32b_x32(trow + c0 * 32, v);
        tmem_ld_wait();
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = 0u;
      }
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const int tok = c0 * 32 + j;
        if (tok < M) part[tok * kDecCols + c_local] = __uint_as_float(v[j]);
      }
    }
  } else {
    *abort_flag = 1;
    raise_status(status, TWELL_ERR_TIMEOUT);
  }
}

// Cluster reduction: CTA `rank` adds the partials of its share of the tokens
// over the cluster's CTAs in rank order (distributed shared memory) and stores
// y once, rounded to bf16.  Every thread of the cluster takes part.
__device__ __forceinline__ void dec_down_reduce(const float *part, uint16_t *y, int M, int d, int split,
                                                uint32_t rank, int col0) {
  __syncwarp();
  cluster_sync();
  const int per = (M + split - 1) / split;
  const int tok0 = static_cast<int>(rank) * per;
  const int ntok = max(0, min(M, tok0 + per) - tok0);
  for (int i = threadIdx.x; i < ntok * (kDecCols / 4); i += blockDim.x) {
    const int tok = tok0 + i / (kDecCols / 4);
    const int c4 = (i % (kDecCols / 4)) * 4;
    const int gc = col0 + c4;
    if (gc >= d) continue;
    const float *src = part + tok * kDecCols + c4;
    float4 acc = ld_shared_cluster_f4(map_to_cta(src, 0));
    for (int r = 1; r < split; ++r) {
      const float4 v = ld_shared_cluster_f4(map_to_cta(src, static_cast<uint32_t>(r)));
      acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
    }
    *reinterpret_cast<uint2 *>(y + static_cast<size_t>(tok) * d + gc) =
        make_uint2(pack_bf16x2(acc.x, acc.y), pack_bf16x2(acc.z, acc.w));
  }
  tc_fence_before();
  __syncwarp();
  cluster_sync();   // no CTA leaves while a peer still reads its partial
  tc_fence_after();
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
    if (lane == 0)
      dec_down_tma(smem, STAGE, kStages, full, empty, abort_flag, &tmap_wd, col0, kb_lo, kb_hi, A.status);
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0)
      dec_down_mma(smem, STAGE, kStages, full, empty, tm_full, drain, abort_flag, tmem_base, P.idesc,
                   kb_hi - kb_lo, A.status);
  } else if (warp < 6) {
    // ------------------------------------------------------------ epilogue: TMEM -> partial
    dec_down_partial(part, tm_full, abort_flag, tmem_base, warp, lane, A.M, true, A.status);
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

  dec_down_reduce(part, P.y, A.M, P.d, P.split, rank, col0);
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem_base, P.tmem_cols);
  }
}

// ============================================================================ touched units
// Bit u of the bitmap is set when some token has h[token][u] != 0: a TwELL slot
// of a pair within ell_w, or a nonzero in the dense backup segment of an
// overflowing pair.  A CTA owns kTouchUnits consecutive hidden units (whole
// tiles, tile_w <= 256) and writes its bitmap words once, so no zeroing pass
// is needed.
constexpr int kTouchUnits = 256;

__global__ void __launch_bounds__(256) k_dec_touch(const TwellView A, uint32_t *bitmap) {
  __shared__ uint32_t words[kTouchUnits / 32];
  griddep_launch_dependents();
  if (threadIdx.x < kTouchUnits / 32) words[threadIdx.x] = 0u;
  __syncthreads();
  griddep_wait();
  const int u0 = blockIdx.x * kTouchUnits;
  const int t0 = u0 / A.tw;
  const int t1 = min(A.T, t0 + kTouchUnits / A.tw);
  const int nt = t1 - t0;
  // pairs within ell_w: their slots
  for (int i = threadIdx.x; i < A.M * nt; i += blockDim.x) {
    const int tok = i / nt, t = t0 + i % nt;
    const size_t pair = static_cast<size_t>(tok) * A.T + t;
    const int n = __ldg(A.nnz + pair);
    if (n > A.E) continue;
    const int ub = t * A.tw - u0;                     // CTA-local unit of in-tile index 0
    const uint8_t *si = A.idx + pair * A.E;
    for (int e = 0; e < n; ++e) {
      const int u = ub + __ldg(si + e);
      if (u < kTouchUnits) atomicOr(&words[u >> 5], 1u << (u & 31));   // in-tile index < tile_w
    }
  }
  // overflowing pairs: the nonzeros of their backup segments (the list is
  // scanned by every CTA; each takes the segments of its own tiles)
  const int n_ovf = min(*A.n_ovf, A.cap);
  const int vec = A.tw / 8;                           // 16-byte pieces per segment
  for (int i = threadIdx.x; i < n_ovf * vec; i += blockDim.x) {
    const int k = i / vec, c8 = (i % vec) * 8;
    const int t = __ldg(A.ovf_pos + k) % A.T;
    if (t < t0 || t >= t1) continue;
    const uint4 q = __ldg(reinterpret_cast<const uint4 *>(A.ovf_dense + static_cast<size_t>(k) * A.tw + c8));
    const uint32_t h[4] = {q.x, q.y, q.z, q.w};
    uint32_t m = 0u;
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if ((h[j >> 1] >> (16 * (j & 1))) & 0x7FFFu) m |= 1u << j;
    if (m != 0u) {
      const int u = t * A.tw - u0 + c8;               // 8 units inside one 32-unit word
      atomicOr(&words[u >> 5], m << (u & 31));
    }
  }
  __syncthreads();
  if (threadIdx.x < kTouchUnits / 32) {
    const int w = u0 / 32 + static_cast<int>(threadIdx.x);
    if (w * 32 < A.f) bitmap[w] = words[threadIdx.x];
  }
}

// Gather mode when at most kGatherNum / kGatherDen of the hidden units are
// touched; above that every W_down row is streamed by TMA as in k_spmm_dec.
constexpr int kGatherNum = 3, kGatherDen = 4;
constexpr int kGatherLag = 4;          // stages a gather thread keeps in flight before signalling one
constexpr size_t kDecTablesOff = 512;  // the lookup tables follow the barrier block

// Split-K down-projection over the touched hidden units only.  Every CTA reads
// the bitmap, scans it (position of each touched unit in the compacted K) and
// lists the units of its share of the compacted K steps.  A K step then holds
// the W_down rows of 64 touched units (gathered by warps 2..5 with 16-byte
// asynchronous copies into the same swizzled operand layout the TMA writes)
// and the h^T columns of the same units (builders map a slot's unit to its
// compacted column).  Untouched rows multiply h columns that are zero for
// every token of the batch, so y is unchanged.
template <int EV>
__global__ void __launch_bounds__(kDecDownThreads, 1)
    k_spmm_dec_touched(const __grid_constant__ CUtensorMap tmap_wd, const DecDownParams P,
                       const uint32_t *__restrict__ bitmap) {
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
  int *scan_s = reinterpret_cast<int *>(bars + 32);        // per-warp totals of the scan
  const TwellView &A = P.A;
  const int W = A.f >> 5;                                  // bitmap words (d_ff % 32 == 0)
  uint32_t *bm_s = reinterpret_cast<uint32_t *>(smem + kStages * STAGE + kDecTablesOff);   // [W + 1]
  int *pre_s = reinterpret_cast<int *>(bm_s + W + 1);      // [W + 1]: touched units before word w
  uint16_t *u_s = reinterpret_cast<uint16_t *>(pre_s + W + 1);   // units of this CTA's share
  float *part = reinterpret_cast<float *>(smem);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int tid = threadIdx.x, nth = blockDim.x;
  const uint32_t rank = cluster_ctarank();
  const int col0 = static_cast<int>(cluster_id_x()) * kDecCols;

  // ---- touched-unit tables (every role needs them; the bitmap comes from the
  // previous kernel)
  griddep_wait();
  const int per = (W + nth - 1) / nth;
  const int w0 = min(W, tid * per), w1 = min(W, w0 + per);
  int cnt = 0;
  for (int w = w0; w < w1; ++w) {
    const uint32_t b = __ldg(bitmap + w);
    bm_s[w] = b;
    cnt += __popc(b);
  }
  int incl = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) scan_s[warp] = incl;
  __syncthreads();
  int run = 0, touched = 0;
  for (int i = 0; i < (nth >> 5); ++i) {
    const int v = scan_s[i];
    if (i < warp) run += v;
    touched += v;
  }
  run += incl - cnt;
  const bool gather = static_cast<long long>(touched) * kGatherDen <= static_cast<long long>(A.f) * kGatherNum;
  for (int w = w0; w < w1; ++w) {
    if (gather) {
      pre_s[w] = run;
      run += __popc(bm_s[w]);
    } else {                                               // every unit in place
      bm_s[w] = 0xFFFFFFFFu;
      pre_s[w] = 32 * w;
    }
  }
  const int Kc = gather ? touched : A.f;                   // compacted K
  if (tid == 0) { bm_s[W] = 0u; pre_s[W] = Kc; }
  __syncthreads();
  const int nsteps = (Kc + kBlockK - 1) / kBlockK;
  const int kb_lo = static_cast<int>((static_cast<long long>(rank) * nsteps) / P.split);
  const int kb_hi = static_cast<int>((static_cast<long long>(rank + 1) * nsteps) / P.split);
  const int p_lo = kb_lo * kBlockK, p_hi = min(kb_hi * kBlockK, Kc);
  const bool has_k = kb_hi > kb_lo;
  if (gather) {
    for (int w = tid; w < W; w += nth) {
      int p = pre_s[w];
      if (pre_s[w + 1] <= p_lo || p >= p_hi) continue;
      uint32_t b = bm_s[w];
      while (b != 0u) {
        const int bit = __ffs(b) - 1;
        b &= b - 1u;
        if (p >= p_lo && p < p_hi) u_s[p - p_lo] = static_cast<uint16_t>(32 * w + bit);
        ++p;
      }
    }
  }
  // unit of compacted column p (p_lo <= p < p_hi); compacted column of touched unit u
  auto unit_at = [&](int p) -> int { return gather ? static_cast<int>(u_s[p - p_lo]) : p; };
  auto pos_of = [&](int u) -> int {
    const int w = u >> 5;
    return pre_s[w] + __popc(bm_s[w] & ((1u << (u & 31)) - 1u));
  };
  auto is_touched = [&](int u) -> bool { return (bm_s[u >> 5] >> (u & 31)) & 1u; };

  // builder warps per step: enough for the operand's np rows (a power of two)
  const int wpg = P.np <= 32 ? 1 : P.np <= 64 ? 2 : P.np <= 128 ? 4 : 8;
  if (tid == 0) {
    // full: the W tile (one TMA arrival with its bytes, or the 4 gather warps)
    // and the wpg builder warps of the step
    for (int i = 0; i < kStages; ++i) { mbar_init(&full[i], (gather ? 4 : 1) + wpg); mbar_init(&empty[i], 1); }
    mbar_init(tm_full, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    if (!gather) tma_prefetch_desc(&tmap_wd);
  }
  if (warp == 1) { tmem_alloc(tmem_slot, P.tmem_cols); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (!gather && lane == 0)
      dec_down_tma(smem, STAGE, kStages, full, empty, abort_flag, &tmap_wd, col0, kb_lo, kb_hi, A.status);
  } else if (warp == 1) {
    if (lane == 0)
      dec_down_mma(smem, STAGE, kStages, full, empty, tm_full, drain, abort_flag, tmem_base, P.idesc,
                   kb_hi - kb_lo, A.status);
  } else if (warp < 6) {
    if (gather) {
      // ---------------------------------------------------------- W_down row gather
      // thread: 16-byte chunk c16 of the 256-byte row piece [col0, col0 + 128),
      // rows r0 + 8 i of the K step; chunk c16 lands in 64-column half c16 / 8
      // at the 128-byte swizzled place of its row
      const int pt = tid - 64;
      const int c16 = pt & 15, r0 = pt >> 4;
      const int gcol = col0 + c16 * 8;
      const bool col_ok = gcol < P.d;
      const uint32_t chunk = static_cast<uint32_t>(c16 & 7);
      const uint32_t half = static_cast<uint32_t>(c16 >> 3) * 8192u;
      int stage = 0; uint32_t phase = 0;
      int issued = 0, sig = 0;                             // groups issued; next stage to signal
      bool ok = true;
      for (int kb = kb_lo; kb < kb_hi; ++kb) {
        if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) { ok = false; break; }
        uint8_t *base = smem + stage * STAGE;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int row = r0 + 8 * i;
          const int p = kb * kBlockK + row;
          const bool live = col_ok && p < p_hi;
          const uint16_t *src = live ? P.w_down + static_cast<size_t>(u_s[p - p_lo]) * P.d + gcol : P.w_down;
          const uint32_t off = half + static_cast<uint32_t>(row) * 128u +
                               ((chunk ^ static_cast<uint32_t>(row & 7)) << 4);
          cp_async_16_zfill(base + off, src, live ? 16u : 0u);
        }
        cp_async_commit();
        if (++issued > kGatherLag) {
          cp_async_wait<kGatherLag>();
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&full[sig]);
          if (++sig == kStages) sig = 0;
        }
        if (++stage == kStages) { stage = 0; phase ^= 1u; }
      }
      cp_async_wait<0>();
      fence_proxy_async_smem();
      __syncwarp();
      for (int i = min(issued, kGatherLag); i > 0; --i) {
        if (lane == 0) mbar_arrive(&full[sig]);
        if (++sig == kStages) sig = 0;
      }
      if (!ok) {
        *abort_flag = 1;
        raise_status(A.status, TWELL_ERR_TIMEOUT);
      }
    }
    dec_down_partial(part, tm_full, abort_flag, tmem_base, warp, lane, A.M, has_k, A.status);
  } else {
    // ------------------------------------------------------------ builders: h^T tiles
    // thread = token row; row i of a stage holds compacted columns
    // [64 kb, 64 kb + 64) of token i, 128-byte swizzled.  A step covers the
    // units [unit_at(64 kb), unit_at(64 kb + 63)], i.e. the tiles between them.
    // The 8 builder warps form 8 / wpg groups of wpg warps (enough warps for
    // the operand's rows); group g builds the steps kb_lo + g + i * groups, so
    // with a few tokens several steps are built at once and the latency of
    // their TwELL record loads overlaps.
    const int bw = warp - 6;
    const int groups = 8 / wpg, grp = bw / wpg;
    const int row = (bw % wpg) * 32 + lane;
    const bool live = row < A.M;
    const bool in_op = row < P.np;                           // the operand has np rows
    const int tw = A.tw, E = A.E, Tn = A.T;
    const int lg_tw = 31 - __clz(tw);
    const int n_ovf = min(*A.n_ovf, A.cap);
    const uint32_t row_swz = static_cast<uint32_t>(row & 7);
    const size_t pair0 = static_cast<size_t>(live ? row : 0) * Tn;
    auto put = [&](uint8_t *rp, int col, uint32_t v) {
      const uint32_t c = static_cast<uint32_t>(col);
      *reinterpret_cast<uint16_t *>(rp + ((((c >> 3) ^ row_swz) << 4) + ((c & 7u) << 1))) = static_cast<uint16_t>(v);
    };
    // the dense backup segment k of tile t: its units in this step, eight
    // loads in flight at a time
    auto put_backup = [&](uint8_t *rp, int t, int k, int p0) {
      const int q_lo = max(p0, pos_of(t << lg_tw));
      const int q_hi = min(min(p0 + kBlockK, p_hi), pos_of((t + 1) << lg_tw));
      const uint16_t *src = A.ovf_dense + static_cast<size_t>(k) * tw - (t << lg_tw);
      for (int q = q_lo; q < q_hi; q += 8) {
        uint32_t v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) v[j] = (q + j < q_hi) ? __ldg(src + unit_at(q + j)) : 0u;
#pragma unroll
        for (int j = 0; j < 8; ++j)
          if (q + j < q_hi) put(rp, q + j - p0, v[j]);
      }
    };
    // this row's backup entries, walked in tile order (a group's tiles only grow)
    int walk = n_ovf;
    if (live && kb_lo + grp < kb_hi)
      walk = ovf_lower_bound(A.ovf_pos, n_ovf, static_cast<int>(pair0) + (unit_at((kb_lo + grp) * kBlockK) >> lg_tw));
    auto find_ovf = [&](int t) -> int {
      while (walk < n_ovf && __ldg(A.ovf_pos + walk) < static_cast<int>(pair0) + t) ++walk;
      return (walk < n_ovf && __ldg(A.ovf_pos + walk) == static_cast<int>(pair0) + t) ? walk : -1;
    };
    // the records of this row's tiles in the CTA's share, asked of L2 up front
    // (group 0 only: the groups share the rows)
    if (live && has_k && grp == 0) {
      const size_t ta = static_cast<size_t>(unit_at(p_lo) >> lg_tw);
      const size_t nt = static_cast<size_t>(unit_at(p_hi - 1) >> lg_tw) - ta + 1;
      prefetch_l2_range(A.vals + (pair0 + ta) * E, nt * E * 2);
      prefetch_l2_range(A.idx + (pair0 + ta) * E, nt * E);
      prefetch_l2_range(A.nnz + pair0 + ta, nt * 2);
    }
    bool ok = true;
    if constexpr (EV > 0) {
      // A tile's record (values, indices, count) is loaded into registers; the
      // first tiles of the group's next step are loaded while this step is
      // built.  A warp walks the tiles together: lane j holds bitmap word j of
      // the tile and the touched units of the tile before it, and a slot's
      // compacted column comes from two shuffles (no per-slot table reads).
      constexpr int EF = 8 * EV;
      constexpr int NPF = EV == 1 ? 2 : 1;                  // tiles of a step loaded ahead
      struct Rec { uint4 v[EV]; uint2 ix[EV]; int n; };
      auto fetch = [&](int t, Rec &r) {
        if (live && t < Tn) {
          const uint4 *gv = reinterpret_cast<const uint4 *>(A.vals + (pair0 + t) * EF);
          const uint2 *gi = reinterpret_cast<const uint2 *>(A.idx + (pair0 + t) * EF);
#pragma unroll
          for (int g = 0; g < EV; ++g) { r.v[g] = __ldg(gv + g); r.ix[g] = __ldg(gi + g); }
          r.n = static_cast<int>(__ldg(A.nnz + pair0 + t));
        } else {
          r.n = 0;
        }
      };
      const int nw = tw >> 5;
      uint32_t t_word = 0u;
      int t_before = 0, t_pos = 0;
      auto tile_map = [&](int t) {                           // warp-uniform
        const int wb = t << (lg_tw - 5);
        t_word = lane < nw ? bm_s[wb + lane] : 0u;
        int c = __popc(t_word);
#pragma unroll
        for (int o = 1; o < 8; o <<= 1) {
          const int v = __shfl_up_sync(0xFFFFFFFFu, c, o);
          if (lane >= o) c += v;
        }
        t_before = c - __popc(t_word);
        t_pos = pre_s[wb];
      };
      auto emit = [&](uint8_t *rp, const Rec &r, int t, int ulo, int uhi, int p0) {
        const bool slots = r.n > 0 && r.n <= EF;
        const int u_t = t << lg_tw;
#pragma unroll
        for (int g = 0; g < EV; ++g) {
          const uint32_t vw[4] = {r.v[g].x, r.v[g].y, r.v[g].z, r.v[g].w};
          const uint32_t iw[2] = {r.ix[g].x, r.ix[g].y};
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int ix = static_cast<int>((iw[e >> 2] >> (8 * (e & 3))) & 0xFFu);
            const uint32_t wj = __shfl_sync(0xFFFFFFFFu, t_word, ix >> 5);
            const int cj = __shfl_sync(0xFFFFFFFFu, t_before, ix >> 5);
            const int u = u_t + ix;
            if (slots && 8 * g + e < r.n && ix < tw && u >= ulo && u <= uhi && ((wj >> (ix & 31)) & 1u))
              put(rp, t_pos + cj + __popc(wj & ((1u << (ix & 31)) - 1u)) - p0, vw[e >> 1] >> (16 * (e & 1)));
          }
        }
        if (r.n > EF) {
          const int k = find_ovf(t);
          if (k >= 0) put_backup(rp, t, k, p0);
        }
      };
      Rec cur[NPF], nxt[NPF];
      int nxt_t0 = -1;
      for (int kb = kb_lo + grp; kb < kb_hi; kb += groups) {
        const int i = kb - kb_lo;
        const int stage = i % kStages;
        const uint32_t par = static_cast<uint32_t>((i / kStages) & 1) ^ 1u;
        const int p0 = kb * kBlockK;
        const int ulo = unit_at(p0), uhi = unit_at(min(p0 + kBlockK, p_hi) - 1);
        const int t_lo = ulo >> lg_tw, t_hi = uhi >> lg_tw;
        if (nxt_t0 == t_lo) {
#pragma unroll
          for (int j = 0; j < NPF; ++j) cur[j] = nxt[j];
        } else {
#pragma unroll
          for (int j = 0; j < NPF; ++j) fetch(t_lo + j, cur[j]);
        }
        nxt_t0 = -1;
        if (kb + groups < kb_hi) {
          nxt_t0 = unit_at((kb + groups) * kBlockK) >> lg_tw;
#pragma unroll
          for (int j = 0; j < NPF; ++j) fetch(nxt_t0 + j, nxt[j]);
        }
        // the lanes leave together (the shuffles need the whole warp)
        if (!__all_sync(0xFFFFFFFFu, mbar_wait(&empty[stage], par, abort_flag))) { ok = false; break; }
        uint8_t *rp = smem + stage * STAGE + kWBytes + row * 128;
        if (in_op) zero_row_128(rp, row);
        for (int t = t_lo; t <= t_hi; ++t) {                 // warp-uniform
          tile_map(t);
          const int j = t - t_lo;
          if (j < NPF) {
#pragma unroll
            for (int jj = 0; jj < NPF; ++jj)
              if (jj == j) emit(rp, cur[jj], t, ulo, uhi, p0);
          } else {
            Rec r;
            fetch(t, r);
            emit(rp, r, t, ulo, uhi, p0);
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&full[stage]);
      }
    } else {
      // any ell_w / tile_w: the row's counts and slots are read per tile
      for (int kb = kb_lo + grp; kb < kb_hi; kb += groups) {
        const int i = kb - kb_lo;
        const int stage = i % kStages;
        const uint32_t par = static_cast<uint32_t>((i / kStages) & 1) ^ 1u;
        const int p0 = kb * kBlockK;
        const int ulo = unit_at(p0), uhi = unit_at(min(p0 + kBlockK, p_hi) - 1);
        if (!__all_sync(0xFFFFFFFFu, mbar_wait(&empty[stage], par, abort_flag))) { ok = false; break; }
        if (in_op) {
          uint8_t *rp = smem + stage * STAGE + kWBytes + row * 128;
          zero_row_128(rp, row);
          if (live) {
            for (int t = ulo >> lg_tw; t <= (uhi >> lg_tw); ++t) {
              const size_t pair = pair0 + t;
              const int n = __ldg(A.nnz + pair);
              if (n == 0) continue;
              if (n <= E) {
                const uint16_t *sv = A.vals + pair * E;
                const uint8_t *si = A.idx + pair * E;
                for (int e = 0; e < n; ++e) {
                  const int u = (t << lg_tw) + __ldg(si + e);
                  if (u >= ulo && u <= uhi && is_touched(u)) put(rp, pos_of(u) - p0, __ldg(sv + e));
                }
              } else {
                const int k = find_ovf(t);
                if (k >= 0) put_backup(rp, t, k, p0);
              }
            }
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&full[stage]);
      }
    }
    if (!ok) {
      *abort_flag = 1;
      raise_status(A.status, TWELL_ERR_TIMEOUT);
    }
  }

  dec_down_reduce(part, P.y, A.M, P.d, P.split, rank, col0);
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

// Batches that take the touched-unit down kernel: TWELL_DECODE_TOUCHED=0 never,
// =all every decode-size batch, unset up to kDecTouchedMaxTokens tokens.  On
// B200 at 4096 -> 16384 and 2 % density it took 36-38 us against 47.6 us for
// the streaming kernel at 32 tokens (about half of W_down's rows touched), but
// 62-72 us against 53 us at 64 tokens (73 % touched), where its builders (one
// group of two warps per K step, four steps in flight) fall behind; the
// streaming kernel can also start reading W_down before the up-projection ends.
constexpr int kDecTouchedMaxTokens = 32;

bool dec_touched_for(int M) {
  static int v = -1;
  if (v < 0) {
    const char *e = getenv("TWELL_DECODE_TOUCHED");
    v = (e == nullptr) ? 1 : (e[0] == '0') ? 0 : (e[0] == 'a') ? 2 : 1;
  }
  return v == 2 || (v == 1 && M <= kDecTouchedMaxTokens);
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

cudaError_t launch_spmm_decode(const TwellView &v, const uint16_t *w_down, int d, uint16_t *y,
                               uint32_t *touch_ws, int num_sms, bool pdl, cudaStream_t s) {
  if (v.M == 0) return cudaSuccess;
  DecDownParams P;
  P.A = v;
  P.w_down = w_down;
  P.y = y;
  P.d = d;
  P.np = round_tokens(v.M);
  P.num_kb = (v.f + kBlockK - 1) / kBlockK;
  P.tmem_cols = tmem_cols_for(P.np);
  P.idesc = idesc_bf16_f32(kDecCols, P.np, 1, 0);
  bool touched = touch_ws != nullptr && dec_touched_for(v.M) && v.f <= 65536;
  const int ev = (v.E % 8 == 0 && v.E <= 64 && v.tw >= 64) ? v.E / 8 : 0;
  void (*kern)(const CUtensorMap, const DecDownParams) = nullptr;
  void (*kern_t)(const CUtensorMap, const DecDownParams, const uint32_t *) = nullptr;
  switch (ev) {
    case 1: kern = k_spmm_dec<1>; kern_t = k_spmm_dec_touched<1>; break;
    case 2: kern = k_spmm_dec<2>; kern_t = k_spmm_dec_touched<2>; break;
    case 3: kern = k_spmm_dec<3>; kern_t = k_spmm_dec_touched<3>; break;
    case 4: kern = k_spmm_dec<4>; kern_t = k_spmm_dec_touched<4>; break;
    case 5: kern = k_spmm_dec<5>; kern_t = k_spmm_dec_touched<5>; break;
    case 6: kern = k_spmm_dec<6>; kern_t = k_spmm_dec_touched<6>; break;
    case 7: kern = k_spmm_dec<7>; kern_t = k_spmm_dec_touched<7>; break;
    case 8: kern = k_spmm_dec<8>; kern_t = k_spmm_dec_touched<8>; break;
    default: kern = k_spmm_dec<0>; kern_t = k_spmm_dec_touched<0>; break;
  }
  // the attribute is the full budget, so the occupancy query below sees the
  // same limit at every token count
  cudaError_t e = cudaFuncSetAttribute(k_spmm_dec<0>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kDecSmemBudget));
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kDecSmemBudget));
  if (e != cudaSuccess) return e;
  if (touched) {
    e = cudaFuncSetAttribute(kern_t, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kDecSmemBudget));
    if (e != cudaSuccess) return e;
  }
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
  // shared memory: stage ring, barrier block, and (touched-unit kernel) the
  // bitmap, its prefix and the unit list of one CTA's share of K
  const size_t stage = static_cast<size_t>(kWBytes) + static_cast<size_t>(P.np) * 128;
  auto ring = [&](size_t tables) -> int {
    const size_t extra = 1024 + kDecTablesOff + ((tables + 15) & ~static_cast<size_t>(15));
    if (extra >= kDecSmemBudget) return 0;
    const size_t n = (kDecSmemBudget - extra) / stage;
    return static_cast<int>(n < static_cast<size_t>(kDecMaxStages) ? n : static_cast<size_t>(kDecMaxStages));
  };
  size_t tables = 0;
  if (touched) {
    const size_t W = static_cast<size_t>(v.f / 32);
    const size_t share = static_cast<size_t>((P.num_kb + best - 1) / best) * kBlockK;
    tables = 8 * (W + 1) + 2 * share;
    // the gather keeps kGatherLag stages in flight before it signals one: with
    // a shorter ring (large batches) every row is streamed instead
    if (ring(tables) <= kGatherLag) { touched = false; tables = 0; }
  }
  const size_t extra = 1024 + kDecTablesOff + ((tables + 15) & ~static_cast<size_t>(15));
  const int stages = ring(tables);
  // the partial [np][128] fp32 reuses the stage buffers
  if (stages < 2 || static_cast<size_t>(stages) * stage < static_cast<size_t>(P.np) * kDecCols * 4)
    return cudaErrorInvalidValue;
  P.stages = stages;
  const size_t smem = extra + stages * stage;
  CUtensorMap mw;
  if (encode_tensor_map_2d(&mw, w_down, d, v.f, static_cast<uint64_t>(d) * 2, 64, kBlockK,
                           CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  if (!touched)
    return launch_k(kern, dim3(n_slices * best), dim3(kDecDownThreads), smem, s, pdl,
                    static_cast<unsigned>(best), mw, P);
  e = launch_k(k_dec_touch, dim3((v.f + kTouchUnits - 1) / kTouchUnits), dim3(256), 0, s, pdl, 1u, v, touch_ws);
  if (e != cudaSuccess) return e;
  return launch_k(kern_t, dim3(n_slices * best), dim3(kDecDownThreads), smem, s, true,
                  static_cast<unsigned>(best), mw, P, static_cast<const uint32_t *>(touch_ws));
}

size_t dec_touch_ws_bytes(int M, int d_ff) {
  return (M > 0 && M <= kDecMaxTokens) ? sizeof(uint32_t) * static_cast<size_t>(d_ff / 32 + 1) : 0;
}

}  // namespace twell
