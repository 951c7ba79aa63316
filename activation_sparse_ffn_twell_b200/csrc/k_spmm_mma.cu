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
// Roles (one CTA per SM, persistent over segments: whole 128-token x 256- or
// 512-column tiles of y, or, on the split schedules, K-step ranges of 512-column
// tiles whose fp32 partials are summed by the last CTA to finish):
//   warp 0      TMA: W_down[k0:k0+64, n0:n0+256] as four 64x64 boxes, 128-byte
//               swizzle; this is an N-major ("MN-major") B operand.  512-column
//               tiles load two such stages per K step from their own ring.
//   warp 1      TMEM allocation (512 fp32 columns: two 256-column accumulators,
//               double-buffered, or both halves of one 512-column tile) +
//               tcgen05.mma issue.
//   warps 2..5  epilogue: TMEM -> fp32 registers -> bf16 -> y (or -> an fp32
//               partial tile, counted at the tile's arrival counter).
//   warps 6..13 A builders.  Fast path (ell_w % 8 == 0): two threads per token
//               row, each taking alternate slots.  The row's slot record of the
//               next hidden tile is in registers (or a TMA-fed shared-memory
//               ring, warp 14) before it is needed; the K steps of one tile are
//               claimed together as soon as the MMA releases them, each thread
//               clears its half of the row, and each slot is written once with
//               a predicated 2-byte store (fully unrolled over ell_w).
//               General path (warps 6..9, thread = row): per K step, zero the
//               row and scatter from global memory.  Then fence to the async
//               proxy and arrive.
//   warp 14     slot producer: TMA boxes of the 128 rows' slot records per
//               hidden tile into the ring.
#include <cstdlib>

#include "twell_device.cuh"

namespace twell {
namespace {

constexpr int kMaxStages = 6;
constexpr int kBN = 256;                        // y columns per tile
constexpr int kABytes = kBlockM * kBlockK * 2;  // 16 KB
constexpr int kBBytes = kBlockK * kBN * 2;      // 32 KB (4 boxes of 64 x 64)
// warps: 0 TMA (W_down), 1 MMA, 2..5 epilogue, 6..13 A builders (two per token
// row on the fast path), 14 slot producer
constexpr int kThreads = 480;
constexpr int kSlotWarp = 14;
constexpr int kSlotRing = 4;                    // max slot-record ring depth (hidden tiles)


struct DownParams {
  TwellView A;
  uint16_t *y;
  int d;
  int num_m_blocks, num_n_blocks, num_kb;
  int stages;                // A pipeline depth (<= kMaxStages), set from shared-memory budget
  int bstages;               // W_down pipeline depth (== stages unless WIDE)
  int slot_ib;               // bytes of the index box per row (covers ell_w indices)
  int ring;                  // slot-record ring depth (2..kSlotRing)
  const int32_t *blk_path;   // NULL, or per 128-token block: 1 = this path owns it
  // Split schedules (512-column tiles, fast builders); a chunk is the K steps
  // of one hidden tile (one K step when tile_w = 32).
  //   1 (split-K): fewer tiles than CTAs.  Tile t's chunks are cut into `parts`
  //     equal ranges; CTA p * tiles + t takes range p, so the CTAs of one range
  //     stream the same W_down rows at the same time.
  //   2 (shared chunks): dp_tiles whole tiles in waves of `grid` (CTA c takes
  //     tiles c, c + grid, ...; none in the current choice), then the other
  //     tiles' chunks dealt out evenly, numbered tile-major, over the first
  //     sk_grid CTAs: CTA c owns chunks [c U / sk_grid, (c + 1) U / sk_grid).
  int split;                 // 0 none, 1 split-K, 2 shared chunks
  int nc, ck;                // chunks per tile, K steps per chunk
  int tiles, parts;          // (1)
  int dp_tiles, sk_grid;     // (2)
  long long units;           // (2) chunks dealt out
  float *part;               // [2 * kMaxSplitCtas][128 x 512] fp32 partial tiles
  int32_t *split_ctr;        // [kMaxSplitCtas] arrivals per shared tile
  int grid;                  // CTAs launched
};

// fp32 partial tile in float4 units: [32-column chunk][8 float4][128 rows], so a
// warp's 32 rows store and load 512 contiguous bytes
constexpr int kPartF4 = kBlockM * 512 / 4;

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
  return P.blk_path == nullptr || P.blk_path[m_blk] == kPathDense;
}

// The schedule helpers below also compile for the host, where
// twell_down_schedule lists a launch's segments without a GPU.
__host__ __device__ __forceinline__ int imin(int a, int b) { return a < b ? a : b; }
__host__ __device__ __forceinline__ long long lmin(long long a, long long b) { return a < b ? a : b; }

// Schedule 2: CTA c owns chunks [c U / G, (c + 1) U / G) of the U dealt out.
__host__ __device__ __forceinline__ long long split_begin(int c, long long U, int G) {
  return static_cast<long long>(c) * U / G;
}
__host__ __device__ __forceinline__ int split_owner(long long q, long long U, int G) {   // CTA of chunk q
  return static_cast<int>(((q + 1) * G + U - 1) / U - 1);
}

// The CTAs that share a tile: `n` of them, the j-th (in K order) is cta(j); each
// publishes its fp32 partial in slot(cta) and the arrivals are counted at ctr.
struct Sharing {
  int n, first, stride, ctr;
  long long ts, U;     // schedule 2: the tile's first dealt chunk, chunks dealt out
  int G;
  __host__ __device__ __forceinline__ Sharing(const DownParams &P, int tile) {
    if (P.split == 1) {
      n = P.parts; first = tile; stride = P.tiles; ctr = tile; ts = 0; U = 0; G = 0;
    } else {
      U = P.units; G = P.sk_grid;
      ts = static_cast<long long>(tile - P.dp_tiles) * P.nc;
      first = split_owner(ts, U, G);
      n = split_owner(ts + P.nc - 1, U, G) - first + 1;
      stride = 1; ctr = first;
    }
  }
  __host__ __device__ __forceinline__ int cta(int j) const { return first + j * stride; }
  // schedule 2: a CTA's segment in this tile is its last one when its share
  // began at or before the tile (slot 2c + 1), else its first one (slot 2c)
  __host__ __device__ __forceinline__ int slot(int c) const {
    return G == 0 ? 2 * c : 2 * c + (split_begin(c, U, G) <= ts ? 1 : 0);
  }
};

// The CTA's work as segments: tile and K steps [kb0, kb1).
struct Sched {
  int mode, c, G, i;
  long long q, qe;
  int tile, kb0, kb1;
  __host__ __device__ __forceinline__ Sched(const DownParams &P, bool split, int unit0, int n_units) {
    mode = split ? P.split : 0;
    c = unit0; G = n_units; i = 0;
    q = qe = 0;
    if (mode == 2 && c < P.sk_grid) {
      q = split_begin(c, P.units, P.sk_grid);
      qe = split_begin(c + 1, P.units, P.sk_grid);
    }
    tile = kb0 = kb1 = 0;
  }
  __host__ __device__ __forceinline__ bool next(const DownParams &P) {
    if (mode == 1) {
      if (i++ > 0) return false;
      tile = c % P.tiles;
      const int p = c / P.tiles;
      kb0 = (p * P.nc / P.parts) * P.ck;
      kb1 = imin(((p + 1) * P.nc / P.parts) * P.ck, P.num_kb);
      return true;
    }
    const int whole_end = mode == 2 ? P.dp_tiles : P.num_m_blocks * P.num_n_blocks;
    const int t = c + i * G;
    if (t < whole_end) {
      ++i;
      tile = t; kb0 = 0; kb1 = P.num_kb;
      return true;
    }
    if (mode != 2 || q >= qe) return false;
    const int r = static_cast<int>(q / P.nc);
    const long long t0 = static_cast<long long>(r) * P.nc;
    const int c0 = static_cast<int>(q - t0);
    const int c1 = static_cast<int>(lmin(qe - t0, static_cast<long long>(P.nc)));
    tile = P.dp_tiles + r;
    kb0 = c0 * P.ck;
    kb1 = imin(c1 * P.ck, P.num_kb);
    q = t0 + c1;
    return true;
  }
};

// EV: ell_w / 8 on the fast builder path, 0 = general path.
// TSLOT: slot records arrive by TMA into a shared-memory ring (else per-thread loads).
// PAIR: a cluster of 2 CTAs computes a 256-token x 256-column tile with M=256
// MMAs (cta_group::2); each CTA builds its 128 rows of A and loads half of the
// W_down columns, so each SM carries half the B operand traffic.
// WIDE (single CTA only): a tile is 128 tokens x 512 y columns -- both halves
// of TMEM -- so each rebuilt A stage feeds two 256-column MMAs, from a separate
// ring of W_down stages.  Half as many A rebuilds per FLOP, and twice the MMA
// time to hide each one behind.  With fast builders it takes the split
// schedules (DownParams::split).
template <int EV, bool TSLOT, bool PAIR, bool WIDE>
__global__ void __launch_bounds__(kThreads, 1)
    k_spmm_mma(const __grid_constant__ CUtensorMap tmap_wd, const __grid_constant__ CUtensorMap tmap_sv,
               const __grid_constant__ CUtensorMap tmap_si, const __grid_constant__ CUtensorMap tmap_sn,
               const DownParams P) {
  static_assert(!(WIDE && PAIR), "512-column tiles are single-CTA");
  constexpr bool SPLIT = WIDE && EV > 0;                      // split schedule compiled in
  constexpr int NH = WIDE ? 2 : 1;                            // 256-column halves per tile
  constexpr int kTN = NH * kBN;                               // y columns per tile
  constexpr int TILE_M = PAIR ? 2 * kBlockM : kBlockM;
  constexpr int B_BYTES = PAIR ? kBBytes / 2 : kBBytes;      // this CTA's W_down columns
  constexpr int B_BOXES = PAIR ? kBN / 128 : kBN / 64;        // 64-column TMA boxes per CTA
  constexpr uint32_t IDESC = idesc_bf16_f32(TILE_M, kBN, 0, 1);
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t *smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  const int kStages = P.stages;
  const int kBStages = P.bstages;
  uint8_t *sA = smem;
  uint8_t *sB = smem + kStages * kABytes;
  uint64_t *bars = reinterpret_cast<uint64_t *>(sB + kBStages * B_BYTES);
  uint64_t *full = bars;
  uint64_t *empty = bars + kMaxStages;
  uint64_t *tm_full = bars + 2 * kMaxStages;
  uint64_t *tm_empty = bars + 2 * kMaxStages + 2;
  uint64_t *drain = bars + 2 * kMaxStages + 4;
  uint64_t *s_full = bars + 2 * kMaxStages + 5;               // slot ring
  uint64_t *s_empty = s_full + kSlotRing;
  uint64_t *bfull = s_empty + kSlotRing;                        // W_down ring (WIDE)
  uint64_t *bempty = bfull + kMaxStages;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bempty + kMaxStages);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  volatile int *split_last = abort_flag + 1;                   // epilogue: last contributor
  // slot ring entry: [128][ell_w] bf16 values, [128][slot_ib] u8 indices, [128][8] u16 nnz
  uint8_t *sRing = reinterpret_cast<uint8_t *>(bars) + 512;
  const int ring_v = kBlockM * 2 * P.A.E, ring_i = kBlockM * P.slot_ib;
  const int ring_entry = ring_v + ring_i + kBlockM * 16;
  const int kRing = P.ring;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const TwellView &A = P.A;

  if (threadIdx.x == 0) {
    constexpr int kBuildWarps = EV > 0 ? 8 : 4;
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full[i], 1 + (PAIR ? 2 : 1) * kBuildWarps);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) { mbar_init(&tm_full[i], 1); mbar_init(&tm_empty[i], PAIR ? 8 : 4); }
    for (int i = 0; i < kSlotRing; ++i) { mbar_init(&s_full[i], 1); mbar_init(&s_empty[i], 8); }
    if (WIDE) for (int i = 0; i < kBStages; ++i) { mbar_init(&bfull[i], 1); mbar_init(&bempty[i], 1); }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmap_wd);
    if (TSLOT) { tma_prefetch_desc(&tmap_sv); tma_prefetch_desc(&tmap_si); tma_prefetch_desc(&tmap_sn); }
  }
  if (warp == 1) {
    if constexpr (PAIR) { tmem_alloc_pair(tmem_slot, 512); tmem_relinquish_pair(); }
    else { tmem_alloc(tmem_slot, 512); tmem_relinquish(); }
  }
  tc_fence_before();
  if constexpr (PAIR) cluster_sync(); else __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // Everything above and the W_down stream (warp 0) depend on no earlier kernel;
  // every other role reads TwELL or writes y, so it waits for the previous
  // kernels of a dependent launch here.
  if (warp != 0) griddep_wait();
  const int num_tiles = P.num_m_blocks * P.num_n_blocks;
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
  const bool leader = rank == 0;
  const int unit0 = PAIR ? static_cast<int>(cluster_id_x()) : static_cast<int>(blockIdx.x);
  const int n_units = PAIR ? static_cast<int>(num_clusters_x()) : static_cast<int>(gridDim.x);
  const int row_base = static_cast<int>(rank) * kBlockM;   // this CTA's rows inside a tile
  const bool split = SPLIT && P.split != 0;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA (W_down)
    if (lane == 0) {
      int stage = 0; uint32_t phase = 0; uint32_t filled = 0;
      int bst = 0; uint32_t bph = 0; uint32_t bfilled = 0;   // W_down ring (WIDE)
      bool ok = true;
      Sched sc(P, split, unit0, n_units);
      while (ok && sc.next(P)) {
        const int tile = sc.tile;
        const int m_blk = tile % P.num_m_blocks, n_blk = tile / P.num_m_blocks;
        if (!tile_owned(P, m_blk * (TILE_M / kBlockM))) continue;
        if constexpr (WIDE) {
          for (int kb = sc.kb0; kb < sc.kb1 && ok; ++kb) {
            if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) { ok = false; break; }
            filled |= 1u << stage;
            mbar_arrive(&full[stage]);   // (no bytes: the builders fill A)
            if (++stage == kStages) { stage = 0; phase ^= 1u; }
            for (int h = 0; h < NH; ++h) {
              if (!mbar_wait(&bempty[bst], bph ^ 1u, abort_flag)) { ok = false; break; }
              mbar_arrive_expect_tx(&bfull[bst], B_BYTES);
              bfilled |= 1u << bst;
              uint8_t *dst = sB + bst * B_BYTES;
              // the 256 columns as four 64-column chunks of one 3-D box
              tma_load_3d(dst, &tmap_wd, &bfull[bst], 0, kb * kBlockK, (n_blk * kTN + h * kBN) / 64);
              if (++bst == kBStages) { bst = 0; bph ^= 1u; }
            }
          }
          continue;
        }
        for (int kb = sc.kb0; kb < sc.kb1; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) { ok = false; break; }
          if (leader) mbar_arrive_expect_tx(&full[stage], (PAIR ? 2 : 1) * B_BYTES);
          filled |= 1u << stage;
          uint8_t *dst = sB + stage * B_BYTES;
          const int col_b = n_blk * kBN + static_cast<int>(rank) * (B_BOXES * 64);
          if constexpr (PAIR) {
#pragma unroll
            for (int j = 0; j < B_BOXES; ++j)
              tma_load_2d_pair(dst + j * (kBlockK * 128), &tmap_wd, map_to_cta(&full[stage], 0),
                               col_b + j * 64, kb * kBlockK);
          } else {   // the tile's 256 columns as four 64-column chunks of one 3-D box
            tma_load_3d(dst, &tmap_wd, &full[stage], 0, kb * kBlockK, col_b / 64);
          }
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) {
        *abort_flag = 1;
        raise_status(A.status, TWELL_ERR_TIMEOUT);
        for (int i = 0; i < kStages; ++i) {
          if (!((filled >> i) & 1u)) continue;
          if (leader && !WIDE) mbar_wait_bounded(&full[i], (i < stage) ? phase : (phase ^ 1u));
        }
        for (int i = 0; WIDE && i < kBStages; ++i) {
          if (!((bfilled >> i) & 1u)) continue;
          mbar_wait_bounded(&bfull[i], (i < bst) ? bph : (bph ^ 1u));
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && leader) {
      int stage = 0; uint32_t phase = 0; int it = 0;
      int bst = 0; uint32_t bph = 0;   // W_down ring (WIDE)
      bool ok = true;
      Sched sc(P, split, unit0, n_units);
      while (ok && sc.next(P)) {
        const int m_blk = sc.tile % P.num_m_blocks;
        if (!tile_owned(P, m_blk * (TILE_M / kBlockM))) continue;
        // WIDE: one accumulator set (both TMEM halves); else two, alternating
        const int acc = WIDE ? 0 : (it & 1);
        const uint32_t acc_phase = WIDE ? (it & 1) : ((it >> 1) & 1);
        ++it;
        if (!mbar_wait<PAIR>(&tm_empty[acc], acc_phase ^ 1u, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kBN);
        if constexpr (WIDE) {
          for (int kb = sc.kb0; kb < sc.kb1 && ok; ++kb) {
            if (!mbar_wait(&full[stage], phase, abort_flag)) { ok = false; break; }
            tc_fence_after();
            const uint32_t a_addr = smem_u32(sA + stage * kABytes);
            for (int h = 0; h < NH; ++h) {
              if (!mbar_wait(&bfull[bst], bph, abort_flag)) { ok = false; break; }
              tc_fence_after();
              const uint32_t b_addr = smem_u32(sB + bst * B_BYTES);
#pragma unroll
              for (int k = 0; k < kBlockK / kUmmaK; ++k) {
                const uint64_t adesc = smem_desc_sw128(a_addr + k * 32, 16, 1024);
                const uint64_t bdesc = smem_desc_sw128(b_addr + k * 2048, kBlockK * 128, 1024);
                umma_bf16(d_tmem + h * kBN, adesc, bdesc, IDESC, (kb != sc.kb0 || k != 0));
              }
              umma_commit(&bempty[bst]);
              if (++bst == kBStages) { bst = 0; bph ^= 1u; }
            }
            umma_commit(&empty[stage]);   // the A stage may be rebuilt
            if (++stage == kStages) { stage = 0; phase ^= 1u; }
          }
          if (!ok) break;
          umma_commit(&tm_full[acc]);
          continue;
        }
        for (int kb = sc.kb0; kb < sc.kb1; ++kb) {
          if (!mbar_wait<PAIR>(&full[stage], phase, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + stage * kABytes);
          const uint32_t b_addr = smem_u32(sB + stage * B_BYTES);
#pragma unroll
          for (int k = 0; k < kBlockK / kUmmaK; ++k) {
            const uint64_t adesc = smem_desc_sw128(a_addr + k * 32, 16, 1024);
            // N-major B: 16 K-rows of 128 B per step; 64-column groups 8 KB apart
            const uint64_t bdesc = smem_desc_sw128(b_addr + k * 2048, kBlockK * 128, 1024);
            if constexpr (PAIR) umma_bf16_pair(d_tmem, adesc, bdesc, IDESC, (kb != sc.kb0 || k != 0));
            else umma_bf16(d_tmem, adesc, bdesc, IDESC, (kb != sc.kb0 || k != 0));
          }
          if constexpr (PAIR) umma_commit_pair_mc(&empty[stage], 0x3);
          else umma_commit(&empty[stage]);
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        if constexpr (PAIR) umma_commit_pair_mc(&tm_full[acc], 0x3);
        else umma_commit(&tm_full[acc]);
      }
      if (!ok) {
        *abort_flag = 1;
        raise_status(A.status, TWELL_ERR_TIMEOUT);
      }
      if constexpr (PAIR) umma_commit_pair_mc(drain, 0x1);
      else umma_commit(drain);
      mbar_wait_bounded(drain, 0);
    }
  } else if (warp == kSlotWarp) {
    // ------------------------------------------------------------ slot producer (TMA)
    if (TSLOT && lane == 0) {
      const int E = A.E;
      const uint32_t bytes = static_cast<uint32_t>(ring_entry);
      int cnt = 0;
      bool ok = true;
      Sched sc(P, split, unit0, n_units);
      while (ok && sc.next(P)) {
        const int m_blk = sc.tile % P.num_m_blocks;
        if (!tile_owned(P, m_blk * (TILE_M / kBlockM))) continue;
        const int r0 = m_blk * TILE_M + row_base;
        // the hidden tiles of the segment's K steps, in the builders' order
        const int t0 = (sc.kb0 * kBlockK) / A.tw;
        const int t1 = min((sc.kb1 * kBlockK + A.tw - 1) / A.tw, A.T);
        for (int t = t0; t < t1; ++t, ++cnt) {
          const int ring = cnt % kRing;
          const uint32_t ph = static_cast<uint32_t>(cnt / kRing) & 1u;
          if (!mbar_wait(&s_empty[ring], ph ^ 1u, abort_flag)) { ok = false; break; }
          mbar_arrive_expect_tx(&s_full[ring], bytes);
          uint8_t *dst = sRing + ring * ring_entry;
          tma_load_2d(dst, &tmap_sv, &s_full[ring], t * E, r0);
          tma_load_2d(dst + ring_v, &tmap_si, &s_full[ring], (t * E) & ~15, r0);
          tma_load_2d(dst + ring_v + ring_i, &tmap_sn, &s_full[ring], t & ~7, r0);
        }
      }
      if (!ok) {
        *abort_flag = 1;
        raise_status(A.status, TWELL_ERR_TIMEOUT);
        for (int i = 0; i < kRing && i < cnt; ++i)   // let issued copies land
          mbar_wait_bounded(&s_full[i], static_cast<uint32_t>((cnt - 1 - ((cnt - 1 - i) % kRing)) / kRing) & 1u);
      }
    }
  } else if (warp < 6) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const int row_in_tile = q * 32 + lane;
    int it = 0;
    Sched sc(P, split, unit0, n_units);
    while (sc.next(P)) {
      const int tile = sc.tile;
      const int m_blk = tile % P.num_m_blocks, n_blk = tile / P.num_m_blocks;
      if (!tile_owned(P, m_blk * (TILE_M / kBlockM))) continue;
      const int acc = WIDE ? 0 : (it & 1);
      const uint32_t acc_phase = WIDE ? (it & 1) : ((it >> 1) & 1);
      ++it;
      bool waited = mbar_wait<PAIR>(&tm_full[acc], acc_phase, abort_flag);
      // one decision per warp (its TMEM loads are warp-wide); with the split
      // schedule one for all four epilogue warps, which meet at barriers below
      waited = __all_sync(0xFFFFFFFFu, waited);
      if (split) waited = !named_bar_any(2, 128, !waited);
      if (!waited) {
        *abort_flag = 1;
        raise_status(A.status, TWELL_ERR_TIMEOUT);
        break;
      }
      tc_fence_after();
      const int r = m_blk * TILE_M + row_base + row_in_tile;
      const bool valid = r < A.M;
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * kBN);
      uint16_t *yr = P.y + static_cast<size_t>(r) * P.d + n_blk * kTN;
      constexpr int NCH = kTN / 32;   // 32-column chunks of the accumulator (8 or 16)
      // bf16 y of chunk c from 32 fp32 words
      auto store_y = [&](const uint32_t (&v)[32], int c) {
        if (valid && n_blk * kTN + c * 32 < P.d) {
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
      };
      // Every chunk pass keeps the next chunk's TMEM load in flight while the
      // current one is converted and stored.
      auto for_chunks = [&](auto &&body) {
        uint32_t va[32], vb[32];
        __syncwarp();
        tmem_ld_32x32b_x32(t_row, va);
        tmem_ld_wait_r32(va);
#pragma unroll 1
        for (int c = 0; c < NCH; c += 2) {
          __syncwarp();
          tmem_ld_32x32b_x32(t_row + (c + 1) * 32, vb);
          body(va, c);
          tmem_ld_wait_r32(vb);
          if (c + 2 < NCH) {
            __syncwarp();
            tmem_ld_32x32b_x32(t_row + (c + 2) * 32, va);
          }
          body(vb, c + 1);
          if (c + 2 < NCH) tmem_ld_wait_r32(va);
        }
      };
      if (!split || (sc.kb0 == 0 && sc.kb1 == P.num_kb)) {
        for_chunks(store_y);
      } else if constexpr (SPLIT) {
        // A tile shared with other CTAs: publish this CTA's fp32 partial, count
        // the arrival, and the last of the contributors adds all partials in K
        // order (0 + p_0 + ... + p_n-1: the same bits whichever CTA finishes
        // last) before the one bf16 rounding.
        const Sharing sh(P, tile);
        const int me = static_cast<int>(blockIdx.x);
        float4 *part = reinterpret_cast<float4 *>(P.part);
        float4 *mine = part + static_cast<size_t>(sh.slot(me)) * kPartF4 + row_in_tile;
        for_chunks([&](const uint32_t (&v)[32], int c) {
#pragma unroll
          for (int j = 0; j < 8; ++j)
            __stcs(mine + (c * 8 + j) * kBlockM,   // streaming: read once, by the finishing CTA
                   make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                               __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3])));
        });
        __threadfence();
        named_bar_sync(2, 128);   // the four epilogue warps
        if (threadIdx.x == 64) {
          const int old = atomicAdd(P.split_ctr + sh.ctr, 1);
          *split_last = (old == sh.n - 1) ? 1 : 0;
        }
        named_bar_sync(2, 128);
        if (*split_last) {
          __threadfence();
          if (sh.n == 2) {
            // Two contributors: fp32 addition is commutative, so own + other
            // has the bits of p_0 + p_1.  The other's next chunk is in flight
            // while the current one is added and stored.
            const int other = sh.cta(0) == me ? sh.cta(1) : sh.cta(0);
            const float4 *src = part + static_cast<size_t>(sh.slot(other)) * kPartF4 + row_in_tile;
            float4 qa[8], qb[8];
            auto add_store = [&](uint32_t (&v)[32], const float4 (&q)[8], int c) {
#pragma unroll
              for (int j = 0; j < 8; ++j) {
                v[4 * j] = __float_as_uint(__uint_as_float(v[4 * j]) + q[j].x);
                v[4 * j + 1] = __float_as_uint(__uint_as_float(v[4 * j + 1]) + q[j].y);
                v[4 * j + 2] = __float_as_uint(__uint_as_float(v[4 * j + 2]) + q[j].z);
                v[4 * j + 3] = __float_as_uint(__uint_as_float(v[4 * j + 3]) + q[j].w);
              }
              store_y(v, c);
            };
#pragma unroll
            for (int j = 0; j < 8; ++j) qa[j] = __ldcs(src + j * kBlockM);
#pragma unroll 1
            for (int c = 0; c < NCH; c += 2) {
#pragma unroll
              for (int j = 0; j < 8; ++j) qb[j] = __ldcs(src + ((c + 1) * 8 + j) * kBlockM);
              uint32_t v[32];
              __syncwarp();
              tmem_ld_32x32b_x32(t_row + c * 32, v);
              tmem_ld_wait_r32(v);
              add_store(v, qa, c);
              if (c + 2 < NCH) {
#pragma unroll
                for (int j = 0; j < 8; ++j) qa[j] = __ldcs(src + ((c + 2) * 8 + j) * kBlockM);
              }
              __syncwarp();
              tmem_ld_32x32b_x32(t_row + (c + 1) * 32, v);
              tmem_ld_wait_r32(v);
              add_store(v, qb, c + 1);
            }
          } else {
#pragma unroll 1
            for (int c = 0; c < NCH; ++c) {
              float s32[32];
#pragma unroll
              for (int j = 0; j < 32; ++j) s32[j] = 0.0f;
              for (int jj = 0; jj < sh.n; ++jj) {
                const int k = sh.cta(jj);
                if (k == me) {
                  uint32_t v[32];
                  __syncwarp();
                  tmem_ld_32x32b_x32(t_row + c * 32, v);
                  tmem_ld_wait_r32(v);
#pragma unroll
                  for (int j = 0; j < 32; ++j) s32[j] += __uint_as_float(v[j]);
                } else {
                  const float4 *src = part + static_cast<size_t>(sh.slot(k)) * kPartF4 +
                                      static_cast<size_t>(c * 8) * kBlockM + row_in_tile;
#pragma unroll
                  for (int j = 0; j < 8; ++j) {
                    const float4 q4 = __ldcs(src + j * kBlockM);
                    s32[4 * j] += q4.x; s32[4 * j + 1] += q4.y; s32[4 * j + 2] += q4.z; s32[4 * j + 3] += q4.w;
                  }
                }
              }
              uint32_t w[32];
#pragma unroll
              for (int j = 0; j < 32; ++j) w[j] = __float_as_uint(s32[j]);
              store_y(w, c);
            }
          }
          if (threadIdx.x == 64) P.split_ctr[sh.ctr] = 0;   // every contributor has arrived
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {   // accumulator free again (the MMAs are issued by the leader)
        if constexpr (PAIR) mbar_arrive_cluster(map_to_cta(&tm_empty[acc], 0));
        else mbar_arrive(&tm_empty[acc]);
      }
    }
  } else if constexpr (EV > 0) {
    // ------------------------------------------------------------ A builders (fast)
    // ell_w == 8*EV.  Per hidden tile, the row's slot record (values, indices,
    // nnz) is in registers before it is needed; the tile's K steps are cleared
    // with independent 16-byte stores and every slot is written once with a
    // predicated 2-byte store -- a fully unrolled, dependency-free sequence.
    constexpr int E = 8 * EV;
    // two threads per token row: `half` takes the slots of its parity
    const int row_in_tile = ((warp - 6) & 3) * 32 + lane;
    const int half = (warp - 6) >> 2;
    const int tw = A.tw, Tn = A.T;
    const int lg_tw = 31 - __clz(tw);
    const int n_ovf = min(*A.n_ovf, A.cap);
    const uint32_t row_swz = static_cast<uint32_t>(row_in_tile & 7);
    int stage = 0; uint32_t phase = 0;
    int scnt = 0;   // slot-ring records consumed so far (TSLOT)
    bool ok = true;
    // The eight builder warps meet at a named barrier once per group of K
    // steps; a bounded wait that gives up is OR-ed into that barrier so they all
    // leave at the same group (no warp is left waiting for the others).
    Sched sc(P, split, unit0, n_units);
    while (sc.next(P)) {
      const int m_blk = sc.tile % P.num_m_blocks;
      if (!tile_owned(P, m_blk * (TILE_M / kBlockM))) continue;
      const int r = m_blk * TILE_M + row_base + row_in_tile;
      const bool valid = r < A.M;
      const size_t pair0 = static_cast<size_t>(valid ? r : 0) * Tn;

      // tile t's slot record of this row, straight into registers
      auto fetch = [&](int t, uint4 (&v)[EV], uint2 (&ix)[EV], int &n) {
        if constexpr (TSLOT) return;                     // the ring path does its own reads
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

      int cur_t = -1, n0 = 0, n1 = 0, ovf_k = -1, ovf_base = -1, ovf_seen = 0;
      uint4 vq[EV], vq1[EV];
      uint2 iq[EV], iq1[EV];
      // K-steps are claimed in groups of S (all steps of one hidden tile when
      // the ring holds them) so every slot is visited once per tile
      // (at most stages-1 of them, so the MMA always has a stage to work on)
      const int S = max(1, min(tw / kBlockK, kStages - 1));
      for (int kb0 = sc.kb0; kb0 < sc.kb1; kb0 += S) {
        const int nsteps = min(S, sc.kb1 - kb0);
        const int stage0 = stage;
        // claim the group's A stages as soon as the MMA has released them and
        // clear this thread's half of its row (row-XOR chunk order: the 32 rows
        // of a warp hit all banks)
        bool fail = !ok;
        for (int j = 0; j < nsteps; ++j) {
          if (!fail && !mbar_wait(&empty[stage], phase ^ 1u, abort_flag)) fail = true;
          if (!fail) {
            uint8_t *rowA = sA + stage * kABytes + row_in_tile * 128;
#pragma unroll
            for (int c = 0; c < 4; ++c)
              *reinterpret_cast<uint4 *>(rowA + (((4 * half + c) ^ static_cast<int>(row_swz)) << 4)) =
                  make_uint4(0u, 0u, 0u, 0u);
          }
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
        fence_proxy_async_smem();   // the zeros precede any backup copy by the async proxy
        if (named_bar_any(1, 256, fail)) { ok = false; break; }
        const int col0 = kb0 * kBlockK, span = nsteps * kBlockK;
        const int t_last = (col0 + span - 1) >> lg_tw;
        for (int t = col0 >> lg_tw; t <= t_last; ++t) {   // 1 tile, or 2 when tile_w == 32
          if (t != cur_t) {                                // same for every thread of the CTA
            if constexpr (TSLOT) {
              // tile t's record waits in ring slot scnt % kRing (filled by TMA)
              const int ring = scnt % kRing;
              if (!mbar_wait(&s_full[ring], static_cast<uint32_t>(scnt / kRing) & 1u, abort_flag)) {
                ok = false;
                break;
              }
              const uint8_t *base_r = sRing + ring * ring_entry;
              const uint8_t *rv = base_r + row_in_tile * (2 * E);
              const uint8_t *ri = base_r + ring_v + row_in_tile * P.slot_ib + ((t * E) & 15);
#pragma unroll
              for (int g = 0; g < EV; ++g) {
                vq[g] = *reinterpret_cast<const uint4 *>(rv + 16 * g);
                iq[g] = *reinterpret_cast<const uint2 *>(ri + 8 * g);
              }
              n0 = (valid && t < Tn)
                       ? static_cast<int>(*reinterpret_cast<const uint16_t *>(
                             base_r + ring_v + ring_i + row_in_tile * 16 + (t & 7) * 2))
                       : 0;
              // the previous slot's values are in registers by now: hand it back
              if (scnt > 0) {
                __syncwarp();
                if (lane == 0) mbar_arrive(&s_empty[(scnt - 1) % kRing]);
              }
              ++scnt;
            } else {
              if (cur_t < 0) {
                fetch(t, vq, iq, n0);
              } else {
#pragma unroll
                for (int g = 0; g < EV; ++g) { vq[g] = vq1[g]; iq[g] = iq1[g]; }
                n0 = n1;
              }
              fetch(t + 1, vq1, iq1, n1);                  // one tile ahead; used next advance
            }
            cur_t = t;
            // backup entry of an overflowing pair: this token's run of entries
            // starts at ovf_base (found once per token), the k-th overflow tile
            // of the row is entry ovf_base + k
            ovf_k = -1;
            if (n0 > E) {
              // (first overflowing tile of the row in this segment: its own entry)
              if (ovf_base < 0) ovf_base = ovf_lower_bound(A.ovf_pos, n_ovf, static_cast<int>(pair0) + t);
              ovf_k = ovf_base + ovf_seen++;
              if (ovf_k >= n_ovf) ovf_k = -1;   // capacity exhausted: y is undefined
            }
          }
          if (!valid || t >= Tn || n0 == 0) continue;
          const int base = (t << lg_tw) - col0;           // group column of in-tile index 0
          if (n0 <= E && base == 0 && span == tw && nsteps <= 2) {
            // the group is exactly this tile (the common case): every slot lands
            // in it, column bit 6 picks the K-step buffer, and the 128-byte
            // swizzle of column c in row r is (2c mod 128) xor 16 (r mod 8)
            int sb1 = stage0 + 1;
            if (sb1 >= kStages) sb1 -= kStages;
            const uint32_t row0 = smem_u32(sA + stage0 * kABytes + row_in_tile * 128);
            const uint32_t row1 = smem_u32(sA + sb1 * kABytes + row_in_tile * 128);
            const uint32_t rsw = row_swz << 4;
#pragma unroll
            for (int g = 0; g < EV; ++g) {
              const uint32_t vw[4] = {vq[g].x, vq[g].y, vq[g].z, vq[g].w};
              const uint32_t iw[2] = {iq[g].x, iq[g].y};
#pragma unroll
              for (int k2 = 0; k2 < 4; ++k2) {   // slot 8g + 2*k2 + half
                const uint32_t cc = 2u * __byte_perm(iw[k2 >> 1], 0u, 0x4440u + 2u * (k2 & 1) + static_cast<uint32_t>(half));
                const uint32_t addr = ((cc & 128u) ? row1 : row0) + ((cc & 127u) ^ rsw);
                if (8 * g + 2 * k2 + half < n0) st_shared_u16(addr, half ? (vw[k2] >> 16) : vw[k2]);
              }
            }
          } else if (n0 <= E) {
            const uint32_t vsh = 16u * static_cast<uint32_t>(half);   // value half of each word
#pragma unroll
            for (int g = 0; g < EV; ++g) {
              const uint32_t vw[4] = {vq[g].x, vq[g].y, vq[g].z, vq[g].w};
              const uint32_t iw[2] = {iq[g].x, iq[g].y};
#pragma unroll
              for (int k2 = 0; k2 < 4; ++k2) {   // slot 8g + 2*k2 + half
                const int sl = 8 * g + 2 * k2 + half;
                const uint32_t ib = (iw[k2 >> 1] >> (16u * (k2 & 1) + 8u * static_cast<uint32_t>(half))) & 0xFFu;
                const uint32_t col = static_cast<uint32_t>(base + static_cast<int>(ib));
                if (sl < n0 && col < static_cast<uint32_t>(span)) {
                  int sb = stage0 + static_cast<int>(col >> 6);   // step buffer of this column
                  if (sb >= kStages) sb -= kStages;
                  const uint32_t c = col & 63u;
                  const uint32_t off = (((c >> 3) ^ row_swz) << 4) + ((c & 7u) << 1);
                  *reinterpret_cast<uint16_t *>(sA + sb * kABytes + row_in_tile * 128 + off) =
                      static_cast<uint16_t>((vw[k2] >> vsh) & 0xFFFFu);
                }
              }
            }
          } else if (ovf_k >= 0) {                        // dense backup segment
            // group columns c with in-tile index c - base inside [0, tile_w)
            const int lo = max(0, base), hi = min(span, base + tw);
            for (int c = lo + 8 * half; c < hi; c += 16) {   // this thread's 16-B chunks
              const uint16_t *src = A.ovf_dense + static_cast<size_t>(ovf_k) * tw + (c - base);
              int sb = stage0 + (c >> 6);
              if (sb >= kStages) sb -= kStages;
              const uint32_t cc = static_cast<uint32_t>(c & 63);
              uint8_t *dst = sA + sb * kABytes + row_in_tile * 128 + (((cc >> 3) ^ row_swz) << 4);
              if constexpr (!PAIR) {
                // async-proxy copy counted on the stage's full barrier: no thread
                // waits for it, and the MMA sees it through that barrier (posted
                // before this warp's arrive, so the phase cannot complete early)
                mbar_expect_tx(&full[sb], 16);
                bulk_load(dst, src, 16, &full[sb]);
              } else {
                *reinterpret_cast<uint4 *>(dst) = __ldg(reinterpret_cast<const uint4 *>(src));
              }
            }
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {   // the MMA (leader CTA) may read these A rows now
          for (int j = 0; j < nsteps; ++j) {
            int sb = stage0 + j;
            if (sb >= kStages) sb -= kStages;
            if constexpr (PAIR) mbar_arrive_cluster(map_to_cta(&full[sb], 0));
            else mbar_arrive(&full[sb]);
          }
        }
      }
      if (!ok) break;   // every builder warp left at the same barrier
    }
    if (!ok) {
      *abort_flag = 1;
      raise_status(A.status, TWELL_ERR_TIMEOUT);
    }
  } else if (warp < 10) {
    // ------------------------------------------------------------ A builders (general)
    // one thread per token row (warps 10..13 idle on this path)
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
  if constexpr (PAIR) cluster_sync(); else __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    if constexpr (PAIR) tmem_dealloc_pair(tmem_base, 512);
    else tmem_dealloc(tmem_base, 512);
  }
}

// Per group of `rows` tokens (128, or 256 when the tensor-core path runs as CTA
// pairs): 1 when its density is at or above the crossover.  The flag is written
// for each 128-token block of the group so both down kernels read one array.
__global__ void __launch_bounds__(256) k_block_path(TwellView A, float crossover, int rows,
                                                    int32_t *blk_path, int32_t *split_ctr) {
  // The next kernel (gather, or the tensor-core kernel with no block flags)
  // reads nothing of this one before its own wait.
  griddep_launch_dependents();
  griddep_wait();   // the counts of the TwELL producer
  // the split schedule's arrival counters start every launch at zero
  if (split_ctr != nullptr && blockIdx.x == 0 && threadIdx.x < kMaxSplitCtas) split_ctr[threadIdx.x] = 0;
  const int blk = blockIdx.x;
  const int r0 = blk * rows;
  const int nr = min(rows, A.M - r0);
  const int n = nr * A.T;                         // counts of the group (<= 256 x 2048)
  const uint16_t *base = A.nnz + static_cast<size_t>(r0) * A.T;
  // the group's counts are contiguous: 16-byte loads (the group starts 16-byte
  // aligned when rows * T is a multiple of 8), a scalar tail, 32-bit sums
  // (at most 256 rows x 2048 tiles x 256)
  const bool vec = ((static_cast<size_t>(r0) * A.T) & 7) == 0;
  const int n8 = vec ? n / 8 : 0;
  uint32_t sum = 0;
  const uint4 *b4 = reinterpret_cast<const uint4 *>(base);
#pragma unroll 4
  for (int i = threadIdx.x; i < n8; i += blockDim.x) {
    const uint4 q = __ldg(b4 + i);
    sum += (q.x & 0xFFFFu) + (q.x >> 16) + (q.y & 0xFFFFu) + (q.y >> 16) +
           (q.z & 0xFFFFu) + (q.z >> 16) + (q.w & 0xFFFFu) + (q.w >> 16);
  }
  for (int i = 8 * n8 + threadIdx.x; i < n; i += blockDim.x) sum += __ldg(base + i);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, o);
  __shared__ uint32_t red[8];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = sum;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t tot = 0;
    for (int w = 0; w < 8; ++w) tot += red[w];
    const double dens = static_cast<double>(tot) / (static_cast<double>(nr) * A.f);
    const int flag = dens >= crossover ? 1 : 0;
    for (int b = r0 / kBlockM; b * kBlockM < r0 + nr; ++b) blk_path[b] = flag;
  }
}

// Split schedule of a 512-column-tile launch (P.num_m_blocks, num_n_blocks,
// num_kb and A set); leaves P.split = 0 when whole tiles are kept.
void plan_split(DownParams &P, int M, int d, int num_sms) {
  const int tw = P.A.tw;
  // Split schedules (512-column tiles, fast builders), chosen so the CTAs that
  // share a tile stay few and the ones streaming W_down stay in step:
  //   fewer tiles than SMs: each tile's K steps cut into `parts` equal ranges
  //     (parts = SMs / tiles, each range at least kMinSplitSteps K steps);
  //   otherwise, unless the tiles fill whole waves: every tile's chunks dealt
  //     out evenly over the SMs.  (Full waves of whole tiles followed by a
  //     shared last wave measured slower on the 2B gated and heavy-tail layers:
  //     per-tile costs differ there, and an even deal of all chunks averages
  //     them out.)
  if (split_ws_bytes(M, d) > 0) {
    constexpr int kMinSplitSteps = 32;
    const int g = num_sms < kMaxSplitCtas ? num_sms : kMaxSplitCtas;
    const int tiles = P.num_m_blocks * P.num_n_blocks;
    P.ck = tw > kBlockK ? tw / kBlockK : 1;
    P.nc = (P.num_kb + P.ck - 1) / P.ck;
    P.tiles = tiles;
    if (tiles < g) {
      int parts = g / tiles;
      const int by_work = (P.nc * P.ck) / kMinSplitSteps;
      if (parts > by_work) parts = by_work;
      if (parts > P.nc) parts = P.nc;
      if (parts >= 2) {
        P.split = 1;
        P.parts = parts;
        P.grid = tiles * parts;
      }
    } else {
      // only when the deal is shorter than the whole-tile waves on every SM, and
      // only for tiles of at least kMinDealSteps K steps: a shared tile costs a
      // partial write and read-back of ~15 us whatever its length.  Measured on
      // B200: 256 tiles of 64 K steps (the backward's weight-gradient products at
      // the 1.5B layer) took longer dealt than whole (backward 0.634 against 0.611
      // ms), 256 tiles of 128 K steps (heavy tail) and 320 of 160 (gated 2B)
      // took less (down 0.353 against 0.402 ms; 0.377 against 0.423 ms).
      constexpr int kMinDealSteps = 128;
      const long long waves = (tiles + num_sms - 1) / num_sms;
      if (tiles % num_sms != 0 && static_cast<long long>(tiles) < waves * g && P.num_kb >= kMinDealSteps) {
        P.dp_tiles = 0;
        P.units = static_cast<long long>(tiles) * P.nc;
        long long sk = (P.units * P.ck) / kMinSplitSteps;
        if (sk > g) sk = g;
        if (sk < 1) sk = 1;
        P.split = 2;
        P.sk_grid = static_cast<int>(sk);
        P.grid = g;
      }
    }
  }
}

template <int EV, bool TSLOT, bool PAIR, bool WIDE = false>
cudaError_t launch_down(const CUtensorMap &mw, const CUtensorMap &sv, const CUtensorMap &si,
                        const CUtensorMap &sn, const DownParams &P, int num_sms, size_t smem,
                        bool pdl, cudaStream_t s) {
  auto kern = k_spmm_mma<EV, TSLOT, PAIR, WIDE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int tiles = P.num_m_blocks * P.num_n_blocks;
  if constexpr (PAIR) {
    // persistent static schedule: only as many pairs as can be resident at once
    static int max_pairs = 0;
    if (max_pairs == 0) {
      cudaLaunchConfig_t cfg = {};
      cfg.blockDim = dim3(kThreads, 1, 1);
      cfg.dynamicSmemBytes = smem;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 2;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      cfg.gridDim = dim3(num_sms & ~1, 1, 1);
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n < 1) n = num_sms / 2;
      max_pairs = n;
    }
    int pairs = max_pairs < num_sms / 2 ? max_pairs : num_sms / 2;
    if (pairs > tiles) pairs = tiles;
    return launch_k(kern, dim3(2 * pairs), dim3(kThreads), smem, s, pdl, 2, mw, sv, si, sn, P);
  } else {
    const int grid = P.split ? P.grid : (tiles < num_sms ? tiles : num_sms);
    return launch_k(kern, dim3(grid), dim3(kThreads), smem, s, pdl, 1, mw, sv, si, sn, P);
  }
}

template <int EV>
cudaError_t launch_down_ev(bool tslot, bool pair, bool wide, const CUtensorMap &mw, const CUtensorMap &sv,
                           const CUtensorMap &si, const CUtensorMap &sn, const DownParams &P,
                           int num_sms, size_t smem, bool pdl, cudaStream_t s) {
  if (wide) {
    if constexpr (EV > 0) {
      if (tslot) return launch_down<EV, true, false, true>(mw, sv, si, sn, P, num_sms, smem, pdl, s);
    }
    return launch_down<EV, false, false, true>(mw, sv, si, sn, P, num_sms, smem, pdl, s);
  }
  if constexpr (EV > 0) {
    if (pair) {
      return tslot ? launch_down<EV, true, true>(mw, sv, si, sn, P, num_sms, smem, pdl, s)
                   : launch_down<EV, false, true>(mw, sv, si, sn, P, num_sms, smem, pdl, s);
    }
    if (tslot) return launch_down<EV, true, false>(mw, sv, si, sn, P, num_sms, smem, pdl, s);
  }
  return launch_down<EV, false, false>(mw, sv, si, sn, P, num_sms, smem, pdl, s);
}

}  // namespace

// CTA-pair mode for this kernel is opt-in (TWELL_DOWN_CTA_PAIR=1): measured on
// the 1.5B layer it is slower than one CTA per tile, because the pair's MMA
// waits for the slower of two builder sets and the builders, not operand
// bandwidth, bound this kernel.
bool down_uses_pair(const TwellView &v) {
  static int env = -1;
  if (env < 0) {
    const char *e = getenv("TWELL_DOWN_CTA_PAIR");
    env = (e != nullptr && e[0] == '1') ? 1 : 0;
  }
  return env == 1 && v.E % 8 == 0 && v.E <= 64;
}

// 512-column tiles are on unless TWELL_DOWN_WIDE=0 (a tuning / comparison knob).
bool down_uses_wide() {
  static int env = -1;
  if (env < 0) {
    const char *e = getenv("TWELL_DOWN_WIDE");
    env = (e != nullptr && e[0] == '0') ? 0 : 1;
  }
  return env == 1;
}

cudaError_t launch_block_path(const TwellView &v, float crossover, int32_t *blk_path, int32_t *split_ctr,
                              bool pdl, cudaStream_t s) {
  const int rows = down_uses_pair(v) ? 2 * kBlockM : kBlockM;
  const int blocks = (v.M + rows - 1) / rows;
  if (blocks == 0) return cudaSuccess;
  return launch_k(k_block_path, dim3(blocks), dim3(256), 0, s, pdl, 1, v, crossover, rows, blk_path,
                  split_ctr);
}

size_t split_ws_bytes(int M, int d_model) {
  if (decode_down_eligible(M) || d_model <= kBN) return 0;
  return 1024 + 2 * static_cast<size_t>(kMaxSplitCtas) * kSplitPartBytes;
}

cudaError_t launch_spmm_mma(const TwellView &v, const uint16_t *w_down, int d, uint16_t *y,
                            const int32_t *blk_path, const SplitWs &split, int num_sms, bool pdl,
                            cudaStream_t s) {
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
  P.split = 0; P.nc = 1; P.ck = 1; P.units = 0; P.grid = 0;
  P.tiles = 0; P.parts = 1; P.dp_tiles = 0; P.sk_grid = 0;
  P.part = split.part; P.split_ctr = split.ctr;
  // Slot records by TMA: the row pitches of vals / idx / nnz must be multiples of
  // 16 bytes and every box start 16-byte aligned (ell_w % 8 == 0, T % 8 == 0).
  const int ib = (v.E % 16 == 0) ? v.E : v.E + 8;
  bool tslot = ev > 0 && v.T % 8 == 0 && (static_cast<long long>(v.T) * v.E) % 16 == 0;
  CUtensorMap sv = mw, si = mw, sn = mw;
  if (tslot) {
    const uint64_t te = static_cast<uint64_t>(v.T) * v.E;
    tslot = encode_tensor_map_2d(&sv, v.vals, te, v.M, te * 2, v.E, kBlockM,
                                 CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_DATA_TYPE_UINT16) == CUDA_SUCCESS &&
            encode_tensor_map_2d(&si, v.idx, te, v.M, te, ib, kBlockM, CU_TENSOR_MAP_SWIZZLE_NONE,
                                 CU_TENSOR_MAP_DATA_TYPE_UINT8) == CUDA_SUCCESS &&
            encode_tensor_map_2d(&sn, v.nnz, v.T, v.M, static_cast<uint64_t>(v.T) * 2, 8, kBlockM,
                                 CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_DATA_TYPE_UINT16) == CUDA_SUCCESS;
  }
  P.slot_ib = ib;
  const bool pair = down_uses_pair(v);
  // single-CTA tiles read W_down through a 3-D view: a box of 64 K-rows x four
  // 64-column chunks lands as the four [64][64] tiles of a 256-column stage in
  // one TMA request (the unit's throughput is bounded per request)
  if (!pair && encode_tensor_map_kchunks(&mw, w_down, d, v.f, kBlockK, 4) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  // 512-column tiles unless y has at most 256 columns (or CTA pairs are on):
  // measured 1.7x the throughput of 256-column tiles per y column, which
  // outweighs a worse-filled last wave of SMs
  const bool wide = !pair && d > kBN && down_uses_wide();
  const int tile_m = pair ? 2 * kBlockM : kBlockM;
  P.num_m_blocks = (v.M + tile_m - 1) / tile_m;
  P.num_n_blocks = (d + (wide ? 2 : 1) * kBN - 1) / ((wide ? 2 : 1) * kBN);
  if (wide && ev > 0 && split.part != nullptr && split.ctr != nullptr) plan_split(P, v.M, d, num_sms);
  const size_t b_stage = pair ? kBBytes / 2 : kBBytes;
  // Pipeline depth from the 227 KB budget.  A deep slot ring (4 hidden tiles)
  // only pays while the pipeline keeps at least 4 stages: at wide ell_w it is
  // cut to 2, which leaves the MMA a free stage while the builders hold a
  // whole hidden tile's K steps.  WIDE: 4 A stages, the rest W_down stages.
  const size_t budget = 227 * 1024;
  int ring_depth = kSlotRing, stages = 0, bstages = 0;
  size_t fixed = 0;
  for (;;) {
    const size_t ring = tslot ? static_cast<size_t>(ring_depth) * kBlockM * (2 * v.E + ib + 16) : 0;
    fixed = 1024 + 512 + ring;
    if (wide) {
      stages = 4;
      bstages = static_cast<int>((budget - fixed - stages * static_cast<size_t>(kABytes)) / b_stage);
      if (bstages > kMaxStages) bstages = kMaxStages;
      if (!tslot || bstages >= 4 || ring_depth == 2) break;
    } else {
      stages = static_cast<int>((budget - fixed) / (kABytes + b_stage));
      if (stages > kMaxStages) stages = kMaxStages;
      bstages = stages;
      if (!tslot || stages >= 4 || ring_depth == 2) break;
    }
    --ring_depth;
  }
  if (stages < 2 || bstages < 2) return cudaErrorInvalidValue;
  P.stages = stages;
  P.bstages = bstages;
  P.ring = ring_depth;
  const size_t smem = fixed + static_cast<size_t>(stages) * kABytes + static_cast<size_t>(bstages) * b_stage;
  switch (ev) {
    case 1: return launch_down_ev<1>(tslot, pair, wide, mw, sv, si, sn, P, num_sms, smem, pdl, s);
    case 2: return launch_down_ev<2>(tslot, pair, wide, mw, sv, si, sn, P, num_sms, smem, pdl, s);
    case 3: return launch_down_ev<3>(tslot, pair, wide, mw, sv, si, sn, P, num_sms, smem, pdl, s);
    case 4: return launch_down_ev<4>(tslot, pair, wide, mw, sv, si, sn, P, num_sms, smem, pdl, s);
    case 5: return launch_down_ev<5>(tslot, pair, wide, mw, sv, si, sn, P, num_sms, smem, pdl, s);
    case 6: return launch_down_ev<6>(tslot, pair, wide, mw, sv, si, sn, P, num_sms, smem, pdl, s);
    case 7: return launch_down_ev<7>(tslot, pair, wide, mw, sv, si, sn, P, num_sms, smem, pdl, s);
    case 8: return launch_down_ev<8>(tslot, pair, wide, mw, sv, si, sn, P, num_sms, smem, pdl, s);
    default: return launch_down_ev<0>(false, false, wide, mw, sv, si, sn, P, num_sms, smem, pdl, s);
  }
}

}  // namespace twell

// Diagnostic: the segments of a tensor-core down-projection launch, computed on
// the host by the same planning and scheduling code the kernel runs.
extern "C" int twell_down_schedule(int M, int d_model, int d_ff, int tile_w, int ell_w, int num_sms,
                                   int32_t *out, int out_len) {
  using namespace twell;
  const bool tw_ok = tile_w == 32 || tile_w == 64 || tile_w == 128 || tile_w == 256;
  if (M <= 0 || d_model <= 0 || d_model % 64 != 0 || d_ff <= 0 || !tw_ok || d_ff % tile_w != 0 ||
      ell_w < 1 || ell_w > tile_w || num_sms <= 0)
    return -1;
  if (decode_down_eligible(M)) return -1;   // the decode-size kernel has its own split
  DownParams P = {};
  P.A.M = M; P.A.f = d_ff; P.A.tw = tile_w; P.A.E = ell_w; P.A.T = d_ff / tile_w;
  if (down_uses_pair(P.A)) return -1;       // the pair grid needs an occupancy query
  const int ev = (ell_w % 8 == 0 && ell_w <= 64) ? ell_w / 8 : 0;
  const bool wide = d_model > kBN && down_uses_wide();
  P.num_m_blocks = (M + kBlockM - 1) / kBlockM;
  P.num_n_blocks = (d_model + (wide ? 2 : 1) * kBN - 1) / ((wide ? 2 : 1) * kBN);
  P.num_kb = (d_ff + kBlockK - 1) / kBlockK;
  P.nc = 1; P.ck = 1; P.parts = 1;
  if (wide && ev > 0) plan_split(P, M, d_model, num_sms);
  const int tiles = P.num_m_blocks * P.num_n_blocks;
  const int grid = P.split ? P.grid : (tiles < num_sms ? tiles : num_sms);
  int n = 0;
  auto put = [&](int v) {
    if (out != nullptr && n < out_len) out[n] = v;
    ++n;
  };
  put(P.split); put(grid); put(tiles); put(P.num_kb);
  for (int c = 0; c < grid; ++c) {
    Sched sc(P, P.split != 0, c, grid);
    while (sc.next(P)) {
      put(c); put(sc.tile); put(sc.kb0); put(sc.kb1);
      if (sc.kb0 == 0 && sc.kb1 == P.num_kb) {
        put(1); put(-1); put(-1);
      } else {
        const Sharing sh(P, sc.tile);
        put(sh.n); put(sh.ctr); put(sh.slot(c));
      }
    }
  }
  return n;
}

