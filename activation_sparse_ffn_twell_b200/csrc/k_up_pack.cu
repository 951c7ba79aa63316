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
//   warp 0      TMA producer: x tile [128 x 64 KCH] and weight tile [256 x 64 KCH]
//               per stage, 128-byte swizzle.  CTA pairs with d_model % 128 == 0
//               take KCH = 2 chunks of 64 K per stage through 3-D tensor maps,
//               so each tile is one 32 KB request instead of two 16 KB ones:
//               measured 110 -> 104.5 us (1.5B layer) and 543 -> 520 us (gated
//               2B layer) for the producer call on one B200.
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
#include <cstdlib>

#include "twell_device.cuh"

namespace twell {
namespace {

constexpr int kThreads = 192;

// PAIR: a cluster of 2 CTAs computes a 256-token tile with M=256 MMAs
// (tcgen05 cta_group::2); each CTA loads its 128 token rows and half of the
// weight rows, so every SM moves half the operand bytes per FLOP.
template <int TW, bool GATED, bool PAIR, int KCH = 1>
struct UpCfg {
  static_assert(KCH == 1 || (KCH == 2 && PAIR), "K chunks per stage: 1, or 2 with CTA pairs");
  static constexpr int A_BYTES = KCH * kBlockM * kBlockK * 2;   // 16 or 32 KB
  static constexpr int N = GATED ? 2 * TW : 256;           // MMA N (accumulator columns)
  static constexpr int TILES_PER_ACC = GATED ? 1 : 256 / TW;
  static constexpr int TILE_M = PAIR ? 2 * kBlockM : kBlockM;
  static constexpr int B_ROWS = PAIR ? N / 2 : N;          // weight rows held by this CTA
  static constexpr int B_BYTES = KCH * B_ROWS * kBlockK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;    // per CTA
  static constexpr int TX_BYTES = (PAIR ? 2 : 1) * STAGE_BYTES;
  static constexpr int STAGES = PAIR ? 6 / KCH : 4;
  static constexpr uint32_t TMEM_COLS = (2 * N <= 32) ? 32 : (2 * N <= 64) ? 64 : (2 * N <= 128) ? 128 : (2 * N <= 256) ? 256 : 512;
  static constexpr uint32_t IDESC = idesc_bf16_f32(TILE_M, N, 0, 0);
};

struct UpParams {
  const uint16_t *b;
  int M, d, f;
  int num_m_blocks, num_n_blocks, num_kb;
  float *z_debug;
  float *l1_part;   // NULL, or [M][T]: per (token, tile) sum of |h| in column order
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

template <int TW, bool GATED, bool PAIR, int KCH>
__global__ void __launch_bounds__(kThreads, 1)
    k_up_pack(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
              const __grid_constant__ CUtensorMap tmap_g, const UpParams P) {
  using C = UpCfg<TW, GATED, PAIR, KCH>;
  constexpr int kStages = C::STAGES;
  griddep_launch_dependents();   // the backup scan waits for this grid anyway
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t *smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);

  uint8_t *sA = smem;                                   // kStages x A_BYTES
  uint8_t *sB = smem + kStages * C::A_BYTES;            // kStages x B_BYTES
  uint8_t *sSlots = sB + kStages * C::B_BYTES;          // 128 rows of slots
  const int E = P.out.E;
  // one 32-bit word per slot (bf16 value | in-tile index << 16); the row pitch is
  // an odd number of words so lanes appending at equal counts hit distinct banks
  const int pitch_w = E + 1 - (E & 1);
  uint32_t *sSlotw = reinterpret_cast<uint32_t *>(sSlots);
  uint64_t *bars = reinterpret_cast<uint64_t *>(
      sSlots + ((static_cast<size_t>(kBlockM) * pitch_w * 4 + 127) & ~static_cast<size_t>(127)));
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
    for (int i = 0; i < 2; ++i) { mbar_init(&tm_full[i], 1); mbar_init(&tm_empty[i], PAIR ? 8 : 4); }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmap_x);
    tma_prefetch_desc(&tmap_w);
    if (GATED) tma_prefetch_desc(&tmap_g);
  }
  if (warp == 1) {
    if constexpr (PAIR) { tmem_alloc_pair(tmem_slot, C::TMEM_COLS); tmem_relinquish_pair(); }
    else { tmem_alloc(tmem_slot, C::TMEM_COLS); tmem_relinquish(); }
  }
  tc_fence_before();
  if constexpr (PAIR) cluster_sync(); else __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int num_tiles = P.num_m_blocks * P.num_n_blocks;
  int32_t *status = P.out.status;
  // work unit = one CTA (or one CTA pair) and its tile stride
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
  const bool leader = rank == 0;
  const int unit0 = PAIR ? static_cast<int>(cluster_id_x()) : static_cast<int>(blockIdx.x);
  const int n_units = PAIR ? static_cast<int>(num_clusters_x()) : static_cast<int>(gridDim.x);

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0; uint32_t phase = 0;
      uint32_t filled = 0;   // bit i: stage i has been filled at least once
      bool ok = true;
      for (int tile = unit0; tile < num_tiles && ok; tile += n_units) {
        const int m_blk = tile % P.num_m_blocks, n_blk = tile / P.num_m_blocks;
        const int a_row = m_blk * C::TILE_M + static_cast<int>(rank) * kBlockM;
        for (int kb = 0; kb < P.num_kb; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) { ok = false; break; }
          // the pair's bytes are all counted on the leader's barrier
          if (leader) mbar_arrive_expect_tx(&full[stage], C::TX_BYTES);
          filled |= 1u << stage;
          uint8_t *a_dst = sA + stage * C::A_BYTES;
          uint8_t *b_dst = sB + stage * C::B_BYTES;
          if constexpr (KCH == 2) {   // (CTA pairs; kb counts stages of 128 K)
            const uint32_t bar = map_to_cta(&full[stage], 0);
            tma_load_3d_pair(a_dst, &tmap_x, bar, 0, a_row, kb * KCH);
            if constexpr (GATED)   // even CTA: gate rows, odd CTA: up rows of the hidden tile
              tma_load_3d_pair(b_dst, rank == 0 ? &tmap_g : &tmap_w, bar, 0, n_blk * TW, kb * KCH);
            else
              tma_load_3d_pair(b_dst, &tmap_w, bar, 0, n_blk * 256 + static_cast<int>(rank) * C::B_ROWS, kb * KCH);
          } else if constexpr (PAIR) {
            const uint32_t bar = map_to_cta(&full[stage], 0);
            tma_load_2d_pair(a_dst, &tmap_x, bar, kb * kBlockK, a_row);
            if constexpr (GATED)   // even CTA: gate rows, odd CTA: up rows of the hidden tile
              tma_load_2d_pair(b_dst, rank == 0 ? &tmap_g : &tmap_w, bar, kb * kBlockK, n_blk * TW);
            else
              tma_load_2d_pair(b_dst, &tmap_w, bar, kb * kBlockK, n_blk * 256 + static_cast<int>(rank) * C::B_ROWS);
          } else {
            tma_load_2d(a_dst, &tmap_x, &full[stage], kb * kBlockK, a_row);
            if constexpr (GATED) {
              tma_load_2d(b_dst, &tmap_g, &full[stage], kb * kBlockK, n_blk * TW);
              tma_load_2d(b_dst + TW * 128, &tmap_w, &full[stage], kb * kBlockK, n_blk * TW);
            } else {
              tma_load_2d(b_dst, &tmap_w, &full[stage], kb * kBlockK, n_blk * 256);
            }
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
        if (leader) {   // (the odd CTA's copies are counted on the leader's barriers)
          for (int i = 0; i < kStages; ++i) {
            if (!((filled >> i) & 1u)) continue;
            const uint32_t par = (i < stage) ? phase : (phase ^ 1u);
            mbar_wait_bounded(&full[i], par);
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && leader) {
      int stage = 0; uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      for (int tile = unit0; tile < num_tiles && ok; tile += n_units, ++it) {
        const int acc = it & 1;
        const uint32_t acc_phase = (it >> 1) & 1;
        if (!mbar_wait<PAIR>(&tm_empty[acc], acc_phase ^ 1u, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * C::N);
        for (int kb = 0; kb < P.num_kb; ++kb) {
          if (!mbar_wait<PAIR>(&full[stage], phase, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + stage * C::A_BYTES);
          const uint32_t b_addr = smem_u32(sB + stage * C::B_BYTES);
#pragma unroll
          for (int k = 0; k < KCH * (kBlockK / kUmmaK); ++k) {   // chunk k / 4: its own [rows][64] tile
            const uint64_t adesc = smem_desc_sw128(a_addr + (k >> 2) * (kBlockM * 128) + (k & 3) * 32, 16, 1024);
            const uint64_t bdesc = smem_desc_sw128(b_addr + (k >> 2) * (C::B_ROWS * 128) + (k & 3) * 32, 16, 1024);
            if constexpr (PAIR) umma_bf16_pair(d_tmem, adesc, bdesc, C::IDESC, (kb | k) != 0);
            else umma_bf16(d_tmem, adesc, bdesc, C::IDESC, (kb | k) != 0);
          }
          if constexpr (PAIR) umma_commit_pair_mc(&empty[stage], 0x3);   // frees the stage in both CTAs
          else umma_commit(&empty[stage]);
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        if constexpr (PAIR) umma_commit_pair_mc(&tm_full[acc], 0x3);
        else umma_commit(&tm_full[acc]);
      }
      if (!ok) {
        *abort_flag = 1;
        raise_status(status, TWELL_ERR_TIMEOUT);
      }
      // all issued MMAs must finish before TMEM is released
      if constexpr (PAIR) umma_commit_pair_mc(drain, 0x1);
      else umma_commit(drain);
      mbar_wait_bounded(drain, 0);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    // The loads and MMAs above read only x and the weights; the epilogue writes
    // the packed output, the staging counters and the status word, which the
    // call's reset kernel zeroes first.
    griddep_wait();
    const int q = warp & 3;                      // TMEM lane quarter of this warp
    const int row_in_tile = q * 32 + lane;
    uint32_t *my_slots = sSlotw + row_in_tile * pitch_w;
    const PackTarget &O = P.out;
    int it = 0;
    for (int tile = unit0; tile < num_tiles; tile += n_units, ++it) {
      const int m_blk = tile % P.num_m_blocks, n_blk = tile / P.num_m_blocks;
      const int acc = it & 1;
      const uint32_t acc_phase = (it >> 1) & 1;
      if (!mbar_wait<PAIR>(&tm_full[acc], acc_phase, abort_flag)) {
        *abort_flag = 1;
        raise_status(status, TWELL_ERR_TIMEOUT);
        break;
      }
      tc_fence_after();
      const int r = m_blk * C::TILE_M + static_cast<int>(rank) * kBlockM + row_in_tile;
      const bool valid = r < P.M;
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * C::N);

#pragma unroll 1
      for (int u = 0; u < C::TILES_PER_ACC; ++u) {
        const int t = GATED ? n_blk : n_blk * C::TILES_PER_ACC + u;
        if (t >= O.T) break;
        const int col0 = t * TW;                 // first hidden column of the tile
        int cnt = 0;
        float l1 = 0.f;                          // sum of |h| over the tile, column order
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
              const bool put = nz && cnt < E;
              l1 += fabsf(__uint_as_float(hb << 16));
              if (__any_sync(0xFFFFFFFFu, put)) {   // no store issued for all-zero columns
                if (put) my_slots[cnt] = hb | (static_cast<uint32_t>(c * 32 + j) << 16);
              }
              cnt += nz ? 1 : 0;
            }
          }
        }
        if (valid) {
          const size_t pair = static_cast<size_t>(r) * O.T + t;
          O.nnz[pair] = static_cast<uint16_t>(cnt);
          if (P.l1_part != nullptr) P.l1_part[pair] = l1;
          uint16_t *gv = O.vals + pair * E;
          uint8_t *gi = O.idx + pair * E;
          if ((E & 7) == 0) {
            for (int s = 0; s < E; s += 8) {   // slots >= cnt are padding: (+0, 0)
              uint32_t w[8];
#pragma unroll
              for (int i = 0; i < 8; ++i) w[i] = (s + i < cnt) ? my_slots[s + i] : 0u;
              *reinterpret_cast<uint4 *>(gv + s) =
                  make_uint4(__byte_perm(w[0], w[1], 0x5410), __byte_perm(w[2], w[3], 0x5410),
                             __byte_perm(w[4], w[5], 0x5410), __byte_perm(w[6], w[7], 0x5410));
              *reinterpret_cast<uint2 *>(gi + s) =
                  make_uint2(__byte_perm(__byte_perm(w[0], w[1], 0x6262), __byte_perm(w[2], w[3], 0x6262), 0x5410),
                             __byte_perm(__byte_perm(w[4], w[5], 0x6262), __byte_perm(w[6], w[7], 0x6262), 0x5410));
            }
          } else {
            for (int s = 0; s < E; ++s) {
              const uint32_t w = (s < cnt) ? my_slots[s] : 0u;
              gv[s] = static_cast<uint16_t>(w & 0xFFFFu);
              gi[s] = static_cast<uint8_t>(w >> 16);
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
      if (lane == 0) {   // the accumulator may be overwritten (MMAs are issued by the leader)
        if constexpr (PAIR) mbar_arrive_cluster(map_to_cta(&tm_empty[acc], 0));
        else mbar_arrive(&tm_empty[acc]);
      }
    }
  }

  tc_fence_before();
  if constexpr (PAIR) cluster_sync(); else __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    if constexpr (PAIR) tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
    else tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

template <int TW, bool GATED, bool PAIR, int KCH>
size_t up_smem_bytes(int E) {
  using C = UpCfg<TW, GATED, PAIR, KCH>;
  const int pitch_w = E + 1 - (E & 1);
  const size_t slots = (static_cast<size_t>(kBlockM) * pitch_w * 4 + 127) & ~static_cast<size_t>(127);
  return 1024 + C::STAGES * (C::A_BYTES + C::B_BYTES) + slots + 256;
}

// CTA pairing is on unless TWELL_UP_CTA_PAIR=0 (a tuning / comparison knob).
bool use_cta_pair() {
  static int v = -1;
  if (v < 0) {
    const char *e = getenv("TWELL_UP_CTA_PAIR");
    v = (e != nullptr && e[0] == '0') ? 0 : 1;
  }
  return v == 1;
}

template <int TW, bool GATED, bool PAIR, int KCH>
cudaError_t launch_up_impl(const UpArgs &a, const PackTarget &t, int num_sms, cudaStream_t s) {
  using C = UpCfg<TW, GATED, PAIR, KCH>;
  CUtensorMap mx, mw, mg;
  const uint32_t w_rows = GATED ? TW : C::B_ROWS;
  auto enc = [&](CUtensorMap *m, const uint16_t *p, int rows, uint32_t box_rows) {
    if constexpr (KCH == 1)
      return encode_tensor_map_2d(m, p, a.d, rows, static_cast<uint64_t>(a.d) * 2, kBlockK, box_rows,
                                  CU_TENSOR_MAP_SWIZZLE_128B);
    else
      return encode_tensor_map_kchunks(m, p, a.d, rows, box_rows, KCH);
  };
  if (enc(&mx, a.x, a.M, kBlockM) != CUDA_SUCCESS) return cudaErrorInvalidValue;
  if (enc(&mw, a.w_up, a.f, w_rows) != CUDA_SUCCESS) return cudaErrorInvalidValue;
  if (GATED) {
    if (enc(&mg, a.w_gate, a.f, TW) != CUDA_SUCCESS) return cudaErrorInvalidValue;
  } else {
    mg = mw;
  }
  UpParams P;
  P.b = a.b;
  P.M = a.M; P.d = a.d; P.f = a.f;
  P.num_m_blocks = (a.M + C::TILE_M - 1) / C::TILE_M;
  P.num_n_blocks = GATED ? t.T : (a.f + 255) / 256;
  P.num_kb = a.d / (KCH * kBlockK);   // pipeline stages per tile
  P.z_debug = a.z_debug;
  P.l1_part = a.l1_part;
  P.out = t;
  const size_t smem = up_smem_bytes<TW, GATED, PAIR, KCH>(t.E);
  cudaError_t e = cudaFuncSetAttribute(k_up_pack<TW, GATED, PAIR, KCH>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int tiles = P.num_m_blocks * P.num_n_blocks;
  if constexpr (PAIR) {
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    // The schedule is persistent and static, so launch only as many pairs as can
    // be resident at once (SM pairing depends on the GPU's cluster layout).
    static int max_pairs = 0;
    if (max_pairs == 0) {
      cfg.gridDim = dim3(num_sms & ~1, 1, 1);
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, k_up_pack<TW, GATED, true, KCH>, &cfg) != cudaSuccess || n < 1)
        n = num_sms / 2;
      max_pairs = n;
    }
    int pairs = max_pairs < num_sms / 2 ? max_pairs : num_sms / 2;
    if (pairs > tiles) pairs = tiles;
    // a dependent launch after the call's reset kernel (see the epilogue's wait)
    return launch_k(k_up_pack<TW, GATED, true, KCH>, dim3(2 * pairs), dim3(kThreads), smem, s, true, 2, mx, mw,
                    mg, P);
  } else {
    const int grid = tiles < num_sms ? tiles : num_sms;
    return launch_k(k_up_pack<TW, GATED, false, KCH>, dim3(grid), dim3(kThreads), smem, s, true, 1, mx, mw, mg, P);
  }
}

template <int TW, bool GATED>
cudaError_t launch_up_sel(const UpArgs &a, const PackTarget &t, int num_sms, cudaStream_t s) {
  if (!use_cta_pair()) return launch_up_impl<TW, GATED, false, 1>(a, t, num_sms, s);
  return a.d % (2 * kBlockK) == 0 ? launch_up_impl<TW, GATED, true, 2>(a, t, num_sms, s)
                                  : launch_up_impl<TW, GATED, true, 1>(a, t, num_sms, s);
}

}  // namespace

cudaError_t launch_up_pack(const UpArgs &a, const PackTarget &t, int num_sms, cudaStream_t s) {
  if (a.M == 0) return cudaSuccess;
  const bool gated = a.w_gate != nullptr;
  switch (t.tw) {
    case 32: return gated ? launch_up_sel<32, true>(a, t, num_sms, s) : launch_up_sel<32, false>(a, t, num_sms, s);
    case 64: return gated ? launch_up_sel<64, true>(a, t, num_sms, s) : launch_up_sel<64, false>(a, t, num_sms, s);
    case 128: return gated ? launch_up_sel<128, true>(a, t, num_sms, s) : launch_up_sel<128, false>(a, t, num_sms, s);
    case 256: return gated ? cudaErrorNotSupported : launch_up_sel<256, false>(a, t, num_sms, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace twell
