// Sparse down-projection on the 2:4 structured-sparse tensor cores.
//
// The down-projection reads only the packed hidden activations (upppp.jp
// 2026-05-11, section 「TwELLとカスタムCUDAカーネルが解決する課題」); on tensor cores
// the pages keep the sparse data aligned to the matmul tiles so the units do not
// idle (innovatopia.jp, editorial notes).  With independent activations a
// 128-token block touches nearly every hidden unit at 1-10 % density, so
// compacting columns saves nothing; what the packed form does give is that a
// token rarely has more than two nonzeros in any 4 consecutive hidden units.
// That is the pattern tcgen05.mma.sp executes at twice the dense rate.
//
// Split of h used here: the hidden units of a tile are cut into aligned groups
// of 4.  In each group the first two nonzeros (ascending unit) go to the 2:4
// operand, the rest -- "excess" -- to a per-token list that the epilogue adds
// on CUDA cores:
//   y = A_2:4 W_down + sum over excess (v * W_down[j])   (fp32, one bf16 rounding)
//
// k_sp_prep (once per call, one warp per token, lanes over hidden tiles) turns
// the TwELL slots (or a pair's dense backup segment) into
//   - the kept values, a [M][d_ff / 2] bf16 matrix laid out for TMA;
//   - their 2-bit position codes, already in the TMEM lane order of the MMA
//     metadata: per 128-token block and 128-unit stage, 128 lanes x 16 bytes;
//   - the excess list of the token, and the token group's down path.
// k_spmm_sp then runs no builders: CTA pairs (cta_group::2), one 256-token x
// 256-column tile of y per pair at a time, persistent over tiles.  Per CTA:
//   warp 0       TMA: the stage's kept values (128 rows x 64) and W_down
//                (128 K-rows x this CTA's 128 columns) as three boxes of 16 KB,
//                completion on the leader.
//   warp 1       TMEM allocation (accumulator columns 0..255, code ring from
//                256) and, on the leader, four M=256 N=256 K=32 sparse MMAs per
//                stage.
//   warps 6..9   position codes: global -> registers -> TMEM (tcgen05.st).
//   warps 2..5, 10..13  epilogue, 128 columns each: TMEM -> fp32, + excess
//                products, -> bf16 y.
//
// Measured on B200 (1.5B layer, 5 %): the sparse MMA itself issues at twice the
// dense rate (M=256 N=256 CTA pairs, operands resident), but this kernel is
// bound by its operand stream: each 128-unit stage moves 96 KB per pair, a
// stage's data lands ~4 us after its loads are issued, and with four 48 KB
// stages in flight per CTA that is ~1 us per stage against ~0.4 us of MMA.
// With the prep pass it takes longer than the dense tensor-core path, so it
// runs only when asked for (TWELL_DOWN_SPARSE).
#include "twell_device.cuh"

namespace twell {
namespace {

constexpr int kSpThreads = 448;                    // 14 warps, roles above
constexpr int kSpBN = 256;                         // y columns per tile
constexpr int kSpABytes = kBlockM * 128;           // kept values of one stage: 128 rows x 64
constexpr int kSpBBox = 128 * 64 * 2;             // W_down box: 128 K-rows x 64 columns (one TMA box)
constexpr int kSpStageBytes = kSpABytes + 2 * kSpBBox;    // 48 KB: kept values + this CTA's 128 columns
constexpr int kSpMaxStages = 4;
constexpr uint32_t kSpMetaCol = 256;               // codes of ring stage i: TMEM columns 256 + 4 i .. + 3

// The operand k_sp_prep writes for k_spmm_sp.
struct SpOperand {
  uint16_t *kept;     // [M][d_ff / 2] kept values
  uint32_t *codes;    // [2 * groups][stages][128 lanes][4] MMA metadata words
  int32_t *xs_cnt;    // [M] excess count per token
  int2 *rowstat;      // [M] (nonzero count, excess count) per token
  float *y_ex;        // [M][d_model] fp32 excess product (tokens with 0 < count <= kSpXc)
  int stages;         // 128-unit stages per token: d_ff / 128
};

struct SpParams {
  TwellView A;
  const uint16_t *w;        // W_down [f][d] (excess rows)
  uint16_t *y;
  int d;
  int num_m_blocks, num_n_blocks;   // 256-token blocks, 256-column blocks
  const int32_t *blk_path;  // per 128-token block: kPathSparse = this kernel
  SpOperand op;
};

__device__ __forceinline__ int find_ovf_sp(const int32_t *pos, int n, int key) {
  int lo = 0, hi = n - 1;
  while (lo <= hi) {
    const int mid = (lo + hi) >> 1;
    const int v = __ldg(pos + mid);
    if (v == key) return mid;
    if (v < key) lo = mid + 1; else hi = mid - 1;
  }
  return -1;
}

__device__ __forceinline__ uint32_t sel4(uint32_t a, uint32_t b, uint32_t c, uint32_t d, int p) {
  return p == 0 ? a : (p == 1 ? b : (p == 2 ? c : d));
}

// Shared-memory scratch of one lane of k_sp_prep (one (token, tile) pair): the
// slot record, the kept values and position codes being built, and the excess.
template <int EV, int TW>
struct alignas(16) PrepLane {
  uint32_t kept[TW / 4];     // TW / 2 kept values
  uint16_t val[8 * EV];
  uint8_t idx[8 * EV];
  uint32_t code[TW / 32];    // one metadata word per MMA of 32 units
  uint32_t xs[kSpXc];        // the pair's excess entries (more than kSpXc: the token's group runs dense)
};
constexpr int kPrepWarps = 8;

// One warp per token (8 per CTA; the grid covers the tokens of whole 256-token
// groups so the codes of padding rows are written too), lane = hidden tile of a
// window of 32.  For each (token, tile) pair: the kept values and position
// codes of its groups of 4 (from the ascending ELL slots, or from the dense
// backup segment of an overflowing pair) and its excess entries.  Then, per
// token: its excess count and list, its nonzero count (rowstat), and -- when
// the list is complete -- the excess product y_ex[r] = sum v * W_down[j] in fp32.
template <int EV, int TW>
__global__ void __launch_bounds__(kPrepWarps * 32) k_sp_prep(TwellView A, const uint16_t *__restrict__ W, int d,
                                                             SpOperand op) {
  constexpr int E = 8 * EV;
  constexpr int KW = TW / 4;          // kept words per pair
  constexpr int NJ = TW / 32;         // MMA words per pair
  using Lane = PrepLane<EV, TW>;
  extern __shared__ __align__(16) uint8_t sm[];
  griddep_launch_dependents();   // the decision kernel reads only after its own wait
  griddep_wait();                // the TwELL producer
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  Lane &L = reinterpret_cast<Lane *>(sm)[warp * 32 + lane];
  const int r = blockIdx.x * kPrepWarps + warp;
  const bool row_ok = r < A.M;
  const int rq = r & (kBlockM - 1);                          // row inside its 128-token block
  const int blk = r / kBlockM;
  const int code_lane = 16 * (rq >> 4) + (rq & 7);           // TMEM lane of units 0..15 of an MMA
  const int code_half = (rq >> 3) & 1;                       // 16-bit half of that lane's word
  const int n_ovf = min(*A.n_ovf, A.cap);
  const size_t pair0 = static_cast<size_t>(row_ok ? r : 0) * A.T;
  // the token's excess list, in tile order (more than kSpXc entries: its group
  // runs on the dense path and the list is not used)
  uint32_t *xs_row = reinterpret_cast<uint32_t *>(sm + sizeof(Lane) * kPrepWarps * 32) + warp * kSpXc;
  uint16_t *codes16 = reinterpret_cast<uint16_t *>(op.codes);
  uint32_t nz = 0;
  int cnt = 0;   // the same in every lane
  for (int t0 = 0; t0 < A.T; t0 += 32) {
    const int t = t0 + lane;
    const bool in = row_ok && t < A.T;
    const int n = in ? static_cast<int>(__ldg(A.nnz + pair0 + t)) : 0;
    nz += static_cast<uint32_t>(n);
    const int n_ell = n <= E ? n : 0;
    if (n_ell > 0) {   // the slot record, for indexed access
      const uint2 *gi = reinterpret_cast<const uint2 *>(A.idx + (pair0 + t) * E);
      const uint4 *gv = reinterpret_cast<const uint4 *>(A.vals + (pair0 + t) * E);
#pragma unroll
      for (int e = 0; e < EV; ++e) {
        reinterpret_cast<uint2 *>(L.idx)[e] = __ldg(gi + e);
        reinterpret_cast<uint4 *>(L.val)[e] = __ldg(gv + e);
      }
    }
#pragma unroll
    for (int c = 0; c < KW / 4; ++c) reinterpret_cast<uint4 *>(L.kept)[c] = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int j = 0; j < NJ; ++j) L.code[j] = 0x44444444u;   // empty group: positions (0, 1)
    uint16_t *kept16 = reinterpret_cast<uint16_t *>(L.kept);
    int my = 0;
    // ELL pairs.  Slots are ascending: a slot is the second of its group when
    // the previous slot is in the same group, excess when the one before is too.
    const int nmax = __reduce_max_sync(0xFFFFFFFFu, static_cast<unsigned>(n_ell));
    int g1 = -1, g2 = -1, p1 = 0;
    for (int sl = 0; sl < nmax; ++sl) {
      if (sl < n_ell) {
        const int i = L.idx[sl] & (TW - 1);
        const uint32_t v = L.val[sl];
        const int grp = i >> 2, p = i & 3;
        const bool nxt_same = sl + 1 < n_ell && ((L.idx[sl + 1] & (TW - 1)) >> 2) == grp;
        if (grp == g2) {
          if (my < kSpXc) L.xs[my] = (static_cast<uint32_t>(t * TW + i) << 16) | v;
          ++my;
        } else {
          const bool second = grp == g1;
          kept16[2 * grp + ((second || (!nxt_same && p == 3)) ? 1 : 0)] = static_cast<uint16_t>(v);
          if (second || !nxt_same) {
            const uint32_t code = second ? static_cast<uint32_t>(p1 | (p << 2))
                                         : (p == 3 ? 0xEu : static_cast<uint32_t>(p | 0xC));
            L.code[grp >> 3] ^= (code ^ 4u) << (4 * (grp & 7));
          }
        }
        g2 = g1;
        g1 = grp;
        p1 = p;
      }
    }
    // Overflowing pairs: the groups of the dense backup segment.
    if (n > E) {
      const int ko = find_ovf_sp(A.ovf_pos, n_ovf, static_cast<int>(pair0 + t));
      if (ko >= 0) {   // (< 0: backup capacity exhausted -- status raised by the producer, y undefined)
        const uint16_t *seg = A.ovf_dense + static_cast<size_t>(ko) * TW;
        for (int j0 = 0; j0 < TW; j0 += 8) {
          const uint4 qv = __ldg(reinterpret_cast<const uint4 *>(seg + j0));
          const uint32_t w4[4] = {qv.x, qv.y, qv.z, qv.w};
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {
            const uint32_t a0 = w4[2 * h2], a1 = w4[2 * h2 + 1];
            const uint32_t v0 = a0 & 0xFFFFu, v1 = a0 >> 16, v2 = a1 & 0xFFFFu, v3 = a1 >> 16;
            const uint32_t m = ((v0 & 0x7FFFu) ? 1u : 0u) | ((v1 & 0x7FFFu) ? 2u : 0u) |
                               ((v2 & 0x7FFFu) ? 4u : 0u) | ((v3 & 0x7FFFu) ? 8u : 0u);
            const int grp = j0 / 4 + h2;
            if (m == 0u) continue;
            const int p0 = __ffs(static_cast<int>(m)) - 1;
            const uint32_t m2 = m & (m - 1u);
            uint32_t comp, code;
            if (m2 == 0u) {
              if (p0 == 3) { comp = v3 << 16; code = 0xEu; }
              else { comp = sel4(v0, v1, v2, v3, p0); code = static_cast<uint32_t>(p0) | 0xCu; }
            } else {
              const int pb = __ffs(static_cast<int>(m2)) - 1;
              comp = sel4(v0, v1, v2, v3, p0) | (sel4(v0, v1, v2, v3, pb) << 16);
              code = static_cast<uint32_t>(p0 | (pb << 2));
              uint32_t rest = m2 & (m2 - 1u);   // nonzeros beyond the first two
              while (rest != 0u) {
                const int px = __ffs(static_cast<int>(rest)) - 1;
                rest &= rest - 1u;
                if (my < kSpXc) L.xs[my] = (static_cast<uint32_t>(t * TW + j0 + 4 * h2 + px) << 16) | sel4(v0, v1, v2, v3, px);
                ++my;
              }
            }
            L.kept[grp] = comp;
            L.code[grp >> 3] ^= (code ^ 4u) << (4 * (grp & 7));
          }
        }
      }
    }
    __syncwarp();
    // position codes -> their TMEM lane order (16-bit halves; rows rq and rq ^ 8
    // share a word), for every stage of the token, padding rows included
    {
      const int sg = ((t0 + lane) * TW) >> 7;             // stage of this tile
      const int jb = (((t0 + lane) * TW) & 127) >> 5;     // its first MMA word in the stage
      if (sg < op.stages) {   // (tiles past the last one have no stage)
        const size_t base = (static_cast<size_t>(blk) * op.stages + sg) * 128;
#pragma unroll
        for (int j = 0; j < NJ; ++j) {
          const uint32_t w = L.code[j];
          codes16[((base + code_lane) * 4 + jb + j) * 2 + code_half] = static_cast<uint16_t>(w & 0xFFFFu);
          codes16[((base + code_lane + 8) * 4 + jb + j) * 2 + code_half] = static_cast<uint16_t>(w >> 16);
        }
      }
    }
    // kept values of the window's tiles, contiguous in the token's row
    if (row_ok) {
      const int ntile = min(32, A.T - t0);
      uint4 *dst = reinterpret_cast<uint4 *>(op.kept + static_cast<size_t>(r) * (A.f / 2) + static_cast<size_t>(t0) * (TW / 2));
      const Lane *lanes = reinterpret_cast<const Lane *>(sm) + warp * 32;
      for (int k = lane; k < ntile * (KW / 4); k += 32)
        dst[k] = reinterpret_cast<const uint4 *>(lanes[k / (KW / 4)].kept)[k % (KW / 4)];
    }
    // excess list: lanes in tile order, each lane's entries ascending
    int incl = my;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
      if (lane >= o) incl += v;
    }
    const int total = __shfl_sync(0xFFFFFFFFu, incl, 31);
    const int off = cnt + incl - my;
    for (int e = 0; e < my && off + e < kSpXc; ++e) xs_row[off + e] = L.xs[e];
    cnt += total;
    __syncwarp();
  }
  const unsigned nz_row = __reduce_add_sync(0xFFFFFFFFu, nz);
  if (row_ok && lane == 0) {
    op.xs_cnt[r] = cnt;
    op.rowstat[r] = make_int2(static_cast<int>(nz_row), cnt);
  }
  // the token's excess product, in fp32, for the 2:4 kernel's epilogue: per
  // entry, the lanes read 8 slices of 256 columns of its W_down row at once
  if (row_ok && cnt > 0 && cnt <= kSpXc) {
    __syncwarp();   // the list written above by every lane of the warp
    const uint32_t mine = lane < cnt ? xs_row[lane] : 0u;
    for (int cb = 0; cb < d; cb += 2048) {
      float acc[8][8];
#pragma unroll
      for (int b = 0; b < 8; ++b)
#pragma unroll
        for (int u = 0; u < 8; ++u) acc[b][u] = 0.f;
      for (int e = 0; e < cnt; ++e) {
        const uint32_t ent = __shfl_sync(0xFFFFFFFFu, mine, e);
        const float hv = __uint_as_float(ent << 16);
        const uint16_t *wrow = W + static_cast<size_t>(ent >> 16) * d;
        uint4 w4[8];
#pragma unroll
        for (int b = 0; b < 8; ++b) {
          const int c0 = cb + b * 256 + lane * 8;
          w4[b] = c0 < d ? __ldg(reinterpret_cast<const uint4 *>(wrow + c0)) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int b = 0; b < 8; ++b) {
          const uint32_t ww[4] = {w4[b].x, w4[b].y, w4[b].z, w4[b].w};
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            acc[b][2 * u] = fmaf(hv, bf16lo_to_f32(ww[u]), acc[b][2 * u]);
            acc[b][2 * u + 1] = fmaf(hv, bf16hi_to_f32(ww[u]), acc[b][2 * u + 1]);
          }
        }
      }
#pragma unroll
      for (int b = 0; b < 8; ++b) {
        const int c0 = cb + b * 256 + lane * 8;
        if (c0 < d) {
          float4 *ye = reinterpret_cast<float4 *>(op.y_ex + static_cast<size_t>(r) * d + c0);
          ye[0] = make_float4(acc[b][0], acc[b][1], acc[b][2], acc[b][3]);
          ye[1] = make_float4(acc[b][4], acc[b][5], acc[b][6], acc[b][7]);
        }
      }
    }
  }
}

// Per 256-token group (one CTA-pair tile of k_spmm_sp): density and the largest
// excess count from the tokens' rowstat, and the group's down path: gather below
// `gather_below`, else the 2:4 kernel when allowed and no token has more than
// kSpXc excess nonzeros, else the dense tensor-core kernel.  Block 0 also
// zeroes the dense kernel's split-schedule counters (split_ctr may be NULL).
__global__ void __launch_bounds__(256) k_sp_decide(const int2 *__restrict__ rowstat, int M, int f, float gather_below,
                                                   int allow_sparse, int32_t *blk_path, int32_t *split_ctr) {
  griddep_launch_dependents();   // the next kernel reads the flags only after its own wait
  griddep_wait();                // the prep's rowstat
  if (split_ctr != nullptr && blockIdx.x == 0 && threadIdx.x < kMaxSplitCtas) split_ctr[threadIdx.x] = 0;
  const int r0 = blockIdx.x * 2 * kBlockM;
  const int nr = min(2 * kBlockM, M - r0);
  int2 st = make_int2(0, 0);
  if (static_cast<int>(threadIdx.x) < nr) st = __ldg(rowstat + r0 + threadIdx.x);
  const unsigned nz = __reduce_add_sync(0xFFFFFFFFu, static_cast<unsigned>(st.x));
  const unsigned xm = __reduce_max_sync(0xFFFFFFFFu, static_cast<unsigned>(st.y));
  __shared__ unsigned s_nz[8], s_xm[8];
  if ((threadIdx.x & 31) == 0) { s_nz[threadIdx.x >> 5] = nz; s_xm[threadIdx.x >> 5] = xm; }
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned long long tot = 0;
    unsigned mx = 0;
    for (int w = 0; w < 8; ++w) { tot += s_nz[w]; mx = max(mx, s_xm[w]); }
    const double dens = static_cast<double>(tot) / (static_cast<double>(nr) * f);
    int flag = kPathDense;
    if (dens < gather_below) flag = kPathGather;
    else if (allow_sparse && mx <= static_cast<unsigned>(kSpXc)) flag = kPathSparse;
    for (int b = r0 / kBlockM; b * kBlockM < r0 + nr; ++b) blk_path[b] = flag;
  }
}

__global__ void __launch_bounds__(kSpThreads, 1)
    k_spmm_sp(const __grid_constant__ CUtensorMap tmap_wd, const __grid_constant__ CUtensorMap tmap_kept,
              const SpParams P) {
  constexpr uint32_t IDESC = idesc_bf16_f32(2 * kBlockM, kSpBN, 0, 1) | (1u << 2);   // sparse
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  uint8_t *smem = smem_raw + (((raw_addr + 1023u) & ~1023u) - raw_addr);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kSpMaxStages * kSpStageBytes);
  uint64_t *full = bars;                     // leader: stage landed + codes stored, both CTAs
  uint64_t *empty = full + kSpMaxStages;     // stage consumed (commit to both CTAs)
  uint64_t *tm_full = empty + kSpMaxStages;  // accumulator complete (commit to both CTAs)
  uint64_t *tm_empty = tm_full + 1;          // leader: accumulator drained, both CTAs (16 warps)
  uint64_t *drain = tm_empty + 1;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const TwellView &A = P.A;
  const int S = P.op.stages;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kSpMaxStages; ++i) { mbar_init(&full[i], 1 + 8); mbar_init(&empty[i], 1); }
    mbar_init(tm_full, 1);
    mbar_init(tm_empty, 16);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmap_wd);
    tma_prefetch_desc(&tmap_kept);
  }
  if (warp == 1) { tmem_alloc_pair(tmem_slot, 512); tmem_relinquish_pair(); }
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  griddep_wait();   // every role reads what the kernels before this one wrote
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int unit0 = static_cast<int>(cluster_id_x());
  const int n_units = static_cast<int>(num_clusters_x());
  const int num_tiles = P.num_m_blocks * P.num_n_blocks;
  auto owned = [&](int m_blk) { return P.blk_path == nullptr || P.blk_path[2 * m_blk] == kPathSparse; };

  if (warp == 0) {
    // ------------------------------------------------------------ TMA
    if (lane == 0) {
      int st = 0;
      uint32_t ph = 0, filled = 0;
      bool ok = true;
      for (int tile = unit0; tile < num_tiles && ok; tile += n_units) {
        const int m_blk = tile % P.num_m_blocks, n_blk = tile / P.num_m_blocks;
        if (!owned(m_blk)) continue;
        const int col = n_blk * kSpBN + static_cast<int>(rank) * 128;
        const int row = m_blk * 2 * kBlockM + static_cast<int>(rank) * kBlockM;
        for (int s = 0; s < S; ++s) {
          if (!mbar_wait(&empty[st], ph ^ 1u, abort_flag)) { ok = false; break; }
          if (leader) mbar_arrive_expect_tx(&full[st], 2 * kSpStageBytes);
          filled |= 1u << st;
          uint8_t *dst = smem + st * kSpStageBytes;
          const uint32_t bar = map_to_cta(&full[st], 0);
          tma_load_2d_pair(dst, &tmap_kept, bar, s * 64, row);
          // (few large boxes: the TMA unit's throughput is bounded per box)
          tma_load_2d_pair(dst + kSpABytes, &tmap_wd, bar, col, s * 128);
          tma_load_2d_pair(dst + kSpABytes + kSpBBox, &tmap_wd, bar, col + 64, s * 128);
          if (++st == kSpMaxStages) { st = 0; ph ^= 1u; }
        }
      }
      if (!ok) {
        *abort_flag = 1;
        raise_status(A.status, TWELL_ERR_TIMEOUT);
        for (int i = 0; leader && i < kSpMaxStages; ++i)   // let issued copies land
          if ((filled >> i) & 1u) mbar_wait_bounded(&full[i], (i < st) ? ph : (ph ^ 1u));
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader)
    if (lane == 0 && leader) {
      int st = 0, it = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int tile = unit0; tile < num_tiles && ok; tile += n_units) {
        if (!owned(tile % P.num_m_blocks)) continue;
        if (!mbar_wait<true>(tm_empty, (it & 1) ^ 1u, abort_flag)) { ok = false; break; }
        ++it;
        tc_fence_after();
        for (int s = 0; s < S; ++s) {
          if (!mbar_wait<true>(&full[st], ph, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + st * kSpStageBytes);
          const uint32_t codes = tmem_base + kSpMetaCol + 4u * static_cast<uint32_t>(st);
#pragma unroll
          for (int mj = 0; mj < 4; ++mj) {   // K = 32 units: kept values 16 mj .. 16 mj + 15
            const uint64_t adesc = smem_desc_sw128(a_addr + mj * 32, 16, 1024);
            // N-major B: 32 K-rows of 128 B per MMA; the two 64-column boxes kSpBBox apart
            const uint64_t bdesc = smem_desc_sw128(a_addr + kSpABytes + mj * 4096, kSpBBox, 1024);
            umma_sp_bf16_pair(tmem_base, adesc, bdesc, IDESC, codes + mj, (s != 0 || mj != 0) ? 1u : 0u);
          }
          umma_commit_pair_mc(&empty[st], 0x3);
          if (++st == kSpMaxStages) { st = 0; ph ^= 1u; }
        }
        if (!ok) break;
        umma_commit_pair_mc(tm_full, 0x3);
      }
      if (!ok) {
        *abort_flag = 1;
        raise_status(A.status, TWELL_ERR_TIMEOUT);
      }
      umma_commit_pair_mc(drain, 0x1);
      mbar_wait_bounded(drain, 0);
    }
  } else if (warp >= 6 && warp < 10) {
    // ------------------------------------------------------------ position codes -> TMEM
    const int q = warp & 3;   // TMEM lane quarter of this warp
    const uint32_t t_lane = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    int st = 0;
    uint32_t ph = 0;
    bool ok = true;
    for (int tile = unit0; tile < num_tiles && ok; tile += n_units) {
      const int m_blk = tile % P.num_m_blocks;
      if (!owned(m_blk)) continue;
      const int blk = 2 * m_blk + static_cast<int>(rank);
      const uint4 *src = reinterpret_cast<const uint4 *>(P.op.codes) + static_cast<size_t>(blk) * S * 128 + 32 * q + lane;
      // a ring of four stages' codes in registers: slot k is reloaded (for stage
      // s + 4) right after stage s used it, so each load has three stages to land
      constexpr int kAhead = 4;
      uint4 cr[kAhead];
#pragma unroll
      for (int k = 0; k < kAhead; ++k) cr[k] = k < S ? __ldg(src + static_cast<size_t>(k) * 128) : make_uint4(0, 0, 0, 0);
      for (int s0 = 0; s0 < S && ok; s0 += kAhead) {
#pragma unroll
        for (int k = 0; k < kAhead; ++k) {
          const int s = s0 + k;
          if (s >= S) break;
          bool w_ok = mbar_wait(&empty[st], ph ^ 1u, abort_flag);
          w_ok = __all_sync(0xFFFFFFFFu, w_ok);
          if (!w_ok) { ok = false; break; }
          tc_fence_after();
          tmem_st_32x32b_x4(t_lane + kSpMetaCol + 4u * static_cast<uint32_t>(st), cr[k].x, cr[k].y, cr[k].z, cr[k].w);
          tmem_st_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(map_to_cta(&full[st], 0));
          if (++st == kSpMaxStages) { st = 0; ph ^= 1u; }
          if (s + kAhead < S) cr[k] = __ldg(src + static_cast<size_t>(s + kAhead) * 128);
        }
      }
    }
    if (!ok) {
      *abort_flag = 1;
      raise_status(A.status, TWELL_ERR_TIMEOUT);
    }
  } else if (warp >= 2) {
    // ------------------------------------------------------------ epilogue (warps 2..5, 10..13)
    const int q = warp & 3;                    // TMEM lane quarter of this warp
    const int c_lo = warp >= 10 ? 4 : 0;       // its four 32-column chunks
    const int row_in_tile = q * 32 + lane;
    int it = 0;
    for (int tile = unit0; tile < num_tiles; tile += n_units) {
      const int m_blk = tile % P.num_m_blocks, n_blk = tile / P.num_m_blocks;
      if (!owned(m_blk)) continue;
      const int r = m_blk * 2 * kBlockM + static_cast<int>(rank) * kBlockM + row_in_tile;
      const bool valid = r < A.M;
      // the token's excess product (fp32, from the prep) when it has excess
      const bool has_ex = valid && __ldg(P.op.xs_cnt + r) > 0;
      const float4 *yex = reinterpret_cast<const float4 *>(P.op.y_ex + static_cast<size_t>(valid ? r : 0) * P.d);
      bool waited = mbar_wait<true>(tm_full, static_cast<uint32_t>(it & 1), abort_flag);
      ++it;
      waited = __all_sync(0xFFFFFFFFu, waited);
      if (!waited) {
        *abort_flag = 1;
        raise_status(A.status, TWELL_ERR_TIMEOUT);
        break;
      }
      tc_fence_after();
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
      uint16_t *yr = P.y + static_cast<size_t>(valid ? r : 0) * P.d;
#pragma unroll 1
      for (int c = c_lo; c < c_lo + 4; ++c) {
        const int col0 = n_blk * kSpBN + c * 32;
        const bool live = valid && col0 < P.d;
        float4 ex[8];
        if (live && has_ex) {
#pragma unroll
          for (int k = 0; k < 8; ++k) ex[k] = __ldg(yex + col0 / 4 + k);
        } else {
#pragma unroll
          for (int k = 0; k < 8; ++k) ex[k] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        uint32_t v[32];
        __syncwarp();
        tmem_ld_32x32b_x32(t_row + c * 32, v);
        tmem_ld_wait_r32(v);
        if (live) {
#pragma unroll
          for (int j = 0; j < 32; j += 8) {
            const float4 a = ex[j / 4], b = ex[j / 4 + 1];
            uint4 o;
            o.x = pack_bf16x2(__uint_as_float(v[j]) + a.x, __uint_as_float(v[j + 1]) + a.y);
            o.y = pack_bf16x2(__uint_as_float(v[j + 2]) + a.z, __uint_as_float(v[j + 3]) + a.w);
            o.z = pack_bf16x2(__uint_as_float(v[j + 4]) + b.x, __uint_as_float(v[j + 5]) + b.y);
            o.w = pack_bf16x2(__uint_as_float(v[j + 6]) + b.z, __uint_as_float(v[j + 7]) + b.w);
            *reinterpret_cast<uint4 *>(yr + col0 + j) = o;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(map_to_cta(tm_empty, 0));
    }
  }

  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc_pair(tmem_base, 512);
  }
}

bool sp_env_enabled() {
  static int v = -1;
  if (v < 0) {
    const char *e = getenv("TWELL_DOWN_SPARSE");
    v = (e != nullptr && e[0] == '0') ? 0 : 1;
  }
  return v == 1;
}

constexpr size_t kSpSmem = 1024 + static_cast<size_t>(kSpMaxStages) * kSpStageBytes + 256;

// Carve-up of the 2:4 path's workspace region.
struct SpWs {
  size_t xs_cnt, rowstat, y_ex, kept, codes, total;
};
SpWs sp_ws_layout(int M, int f, int d) {
  SpWs w;
  const size_t groups = (static_cast<size_t>(M) + 2 * kBlockM - 1) / (2 * kBlockM);
  const size_t stages = static_cast<size_t>(f) / 128;
  size_t o = 0;
  w.xs_cnt = o;  o = align256(o + sizeof(int32_t) * static_cast<size_t>(M));
  w.rowstat = o; o = align256(o + sizeof(int2) * static_cast<size_t>(M));
  w.y_ex = o;    o = align256(o + sizeof(float) * static_cast<size_t>(M) * d);
  w.kept = o;    o = align256(o + 2 * static_cast<size_t>(M) * (f / 2));
  w.codes = o;   o = align256(o + groups * 2 * stages * 128 * 16);
  w.total = o;
  return w;
}

SpOperand sp_operand(void *ws, int M, int f, int d) {
  const SpWs L = sp_ws_layout(M, f, d);
  uint8_t *b = static_cast<uint8_t *>(ws);
  SpOperand op;
  op.xs_cnt = reinterpret_cast<int32_t *>(b + L.xs_cnt);
  op.rowstat = reinterpret_cast<int2 *>(b + L.rowstat);
  op.y_ex = reinterpret_cast<float *>(b + L.y_ex);
  op.kept = reinterpret_cast<uint16_t *>(b + L.kept);
  op.codes = reinterpret_cast<uint32_t *>(b + L.codes);
  op.stages = f / 128;
  return op;
}

template <int EV, int TW>
cudaError_t launch_prep_impl(const TwellView &v, const uint16_t *w_down, int d, const SpOperand &op, bool pdl,
                             cudaStream_t s) {
  const int groups = (v.M + 2 * kBlockM - 1) / (2 * kBlockM);
  const size_t smem = sizeof(PrepLane<EV, TW>) * kPrepWarps * 32 + sizeof(uint32_t) * kPrepWarps * kSpXc;
  cudaError_t e = cudaFuncSetAttribute(k_sp_prep<EV, TW>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int blocks = groups * 2 * kBlockM / kPrepWarps;   // whole groups: padding rows get their codes
  return launch_k(k_sp_prep<EV, TW>, dim3(blocks), dim3(kPrepWarps * 32), smem, s, pdl, 1, v, w_down, d, op);
}

}  // namespace

bool sp_eligible(const TwellView &v, int d) {
  return sp_env_enabled() && (v.tw == 128 || v.tw == 64) && v.E % 8 == 0 && v.E <= 32 && v.f < 65536 &&
         v.f % 128 == 0 && d > 0 && d % 64 == 0 && !decode_down_eligible(v.M);
}

size_t sp_ws_bytes(int M, int d_ff, int d_model) { return sp_ws_layout(M, d_ff, d_model).total; }

cudaError_t launch_sp_prep(const TwellView &v, const uint16_t *w_down, int d, void *sp_ws, float gather_below,
                           bool allow_sparse, int32_t *blk_path, int32_t *split_ctr, bool pdl, cudaStream_t s) {
  if (v.M == 0) return cudaSuccess;
  if (!sp_eligible(v, d)) return cudaErrorInvalidValue;
  const SpOperand op = sp_operand(sp_ws, v.M, v.f, d);
  const int ev = v.E / 8;
  const bool t64 = v.tw == 64;
  cudaError_t e;
  switch (ev) {
    case 1: e = t64 ? launch_prep_impl<1, 64>(v, w_down, d, op, pdl, s) : launch_prep_impl<1, 128>(v, w_down, d, op, pdl, s); break;
    case 2: e = t64 ? launch_prep_impl<2, 64>(v, w_down, d, op, pdl, s) : launch_prep_impl<2, 128>(v, w_down, d, op, pdl, s); break;
    case 3: e = t64 ? launch_prep_impl<3, 64>(v, w_down, d, op, pdl, s) : launch_prep_impl<3, 128>(v, w_down, d, op, pdl, s); break;
    case 4: e = t64 ? launch_prep_impl<4, 64>(v, w_down, d, op, pdl, s) : launch_prep_impl<4, 128>(v, w_down, d, op, pdl, s); break;
    default: return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess) return e;
  const int groups = (v.M + 2 * kBlockM - 1) / (2 * kBlockM);
  return launch_k(k_sp_decide, dim3(groups), dim3(256), 0, s, true, 1, static_cast<const int2 *>(op.rowstat), v.M,
                  v.f, gather_below, allow_sparse ? 1 : 0, blk_path, split_ctr);
}

cudaError_t launch_spmm_sp(const TwellView &v, const uint16_t *w_down, int d, uint16_t *y, const int32_t *blk_path,
                           void *sp_ws, int num_sms, bool pdl, cudaStream_t s) {
  if (v.M == 0) return cudaSuccess;
  if (!sp_eligible(v, d)) return cudaErrorInvalidValue;
  SpParams P;
  P.A = v;
  P.w = w_down;
  P.y = y;
  P.d = d;
  P.num_m_blocks = (v.M + 2 * kBlockM - 1) / (2 * kBlockM);
  P.num_n_blocks = (d + kSpBN - 1) / kSpBN;
  P.blk_path = blk_path;
  P.op = sp_operand(sp_ws, v.M, v.f, d);
  CUtensorMap mw, mk;
  if (encode_tensor_map_2d(&mw, w_down, d, v.f, static_cast<uint64_t>(d) * 2, 64, 128,
                           CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  if (encode_tensor_map_2d(&mk, P.op.kept, v.f / 2, v.M, static_cast<uint64_t>(v.f / 2) * 2, 64, kBlockM,
                           CU_TENSOR_MAP_SWIZZLE_128B) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(k_spmm_sp, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kSpSmem));
  if (e != cudaSuccess) return e;
  static int max_pairs = 0;   // persistent static schedule: only pairs that can be resident at once
  if (max_pairs == 0) {
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(kSpThreads, 1, 1);
    cfg.dynamicSmemBytes = kSpSmem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cfg.gridDim = dim3(num_sms & ~1, 1, 1);
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, k_spmm_sp, &cfg) != cudaSuccess || n < 1) n = num_sms / 2;
    max_pairs = n;
  }
  const int tiles = P.num_m_blocks * P.num_n_blocks;
  int pairs = max_pairs < num_sms / 2 ? max_pairs : num_sms / 2;
  if (pairs > tiles) pairs = tiles;
  if (pairs < 1) pairs = 1;
  return launch_k(k_spmm_sp, dim3(2 * pairs), dim3(kSpThreads), kSpSmem, s, pdl, 2, mw, mk, P);
}

}  // namespace twell
