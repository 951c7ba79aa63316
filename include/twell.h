/*
 * twell.h -- C ABI of the B200 (sm_100a) activation-sparse FFN library.
 *
 * The operation is the forward pass of a ReLU feed-forward layer whose hidden
 * activations are mostly zero: an up-projection to a wide hidden dimension, a
 * ReLU, and a down-projection back to the model dimension, tokens independent
 * ("Sparser, Faster, Lighter Transformer Language Models", Sakana AI / NVIDIA;
 * upppp.jp 2026-05-11, section 「LLMフィードフォワード層の「無駄」とは何か」).
 * The hidden activations are packed into TwELL (Tile-wise ELLPACK): hidden
 * columns are cut into fixed-width tiles and, per token and tile, an ELL list of
 * (value, in-tile index) slots keeps the nonzeros; (token, tile) pairs with more
 * nonzeros than the ELL width also keep their dense tile segment in a small dense
 * backup -- the "hybrid" sparse-main plus dense-backup form (same page, section
 * 「TwELLとカスタムCUDAカーネルが解決する課題」).  The down-projection reads only
 * the packed form.
 *
 * Conventions for every call
 *  - bf16 tensors are passed as uint16_t bit patterns.  All tensor pointers are
 *    DEVICE pointers, caller-owned, 16-byte aligned, row-major and dense unless a
 *    leading dimension says otherwise.  The library allocates no device memory;
 *    scratch comes from the caller's workspace (see twell_workspace_bytes).
 *  - `stream` is a cudaStream_t (NULL = legacy default stream).  Calls are
 *    asynchronous: they validate arguments on the host, enqueue kernels and
 *    return.  Argument errors are returned before anything is enqueued.
 *  - Asynchronous errors (backup capacity exhausted, a bounded device wait that
 *    timed out) are recorded in the matrix's device status word; read them with
 *    twell_read_status, which synchronises the stream.
 *  - Shapes: tile_w in {32, 64, 128, 256}; d_ff % tile_w == 0;
 *    1 <= ell_w <= tile_w; d_model % 64 == 0; M >= 0 (M == 0 is a no-op).
 */
#ifndef TWELL_B200_H
#define TWELL_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  TWELL_OK = 0,
  TWELL_ERR_INVALID_ARG = 1,      /* null/misaligned pointer, bad shape            */
  TWELL_ERR_UNSUPPORTED = 2,      /* legal but not implemented (e.g. gated tile_w 256) */
  TWELL_ERR_OVERFLOW_CAPACITY = 3,/* async: more overflow pairs than ovf_capacity   */
  TWELL_ERR_CUDA = 4,             /* a CUDA runtime/driver call failed               */
  TWELL_ERR_TIMEOUT = 5,          /* async: a bounded device wait gave up            */
  TWELL_ERR_WORKSPACE = 6         /* workspace missing or smaller than required      */
} twell_status;

/* Down-projection path selection. */
typedef enum {
  TWELL_DOWN_AUTO = 0,   /* per 128-token block, by measured density crossover:
                            GATHER below it, MMA at or above it                   */
  TWELL_DOWN_GATHER = 1, /* CUDA-core gather of W_down rows per packed nonzero    */
  TWELL_DOWN_MMA = 2,    /* tcgen05 tensor cores on h tiles rebuilt from TwELL.
                            AUTO and MMA with M <= 256 take the decode-size
                            split-K kernel (tokens on the MMA's N side); up to
                            32 tokens it runs on the hidden units some token
                            uses, reading only their W_down rows                */
  TWELL_DOWN_SPARSE = 3  /* tcgen05 2:4 structured-sparse tensor cores: per group
                            of 4 hidden units the first two nonzeros run on the
                            sparse MMA, the rest are added on CUDA cores.  Taken
                            per 256-token group when every token has at most 32
                            such extra nonzeros (else MMA); tile_w 64 or 128,
                            ell_w % 8 == 0 and <= 32, d_ff % 128 == 0, M > 256
                            (other shapes run MMA).  Explicit only: on B200 it
                            measured slower than MMA at every density.            */
} twell_down_mode;

/*
 * A TwELL matrix of M tokens x d_ff hidden units (T = d_ff / tile_w tiles).
 *   vals      [M][T][ell_w]  bf16  slot values; unused slots hold +0
 *   idx       [M][T][ell_w]  u8    in-tile column of each slot (unused: 0)
 *   nnz       [M][T]         u16   TRUE nonzero count of the pair (may exceed ell_w)
 *   n_ovf     [1]            i32   number of pairs with nnz > ell_w (true count)
 *   ovf_pos   [ovf_capacity] i32   r*T + t of each overflowing pair, ascending
 *   ovf_dense [ovf_capacity][tile_w] bf16  the pair's whole dense tile segment
 *   status    [1]            i32   0, or a twell_status raised on the device
 * Slots list a pair's nonzeros in ascending in-tile order; "nonzero" means the
 * bf16 value is not +-0, and every stored zero is +0.  For an overflowing pair the
 * slots still hold its first ell_w nonzeros; consumers use the dense segment.
 * All arrays are device memory owned by the caller.
 */
typedef struct {
  int32_t M, d_ff, tile_w, ell_w;
  uint16_t *vals;
  uint8_t *idx;
  uint16_t *nnz;
  int32_t ovf_capacity;
  int32_t *n_ovf;
  int32_t *ovf_pos;
  uint16_t *ovf_dense;
  int32_t *status;
} twell_matrix;

/* Library version (major*10000 + minor*100 + patch). */
int twell_version(void);

/* Human-readable name of a status code (static string). */
const char *twell_status_string(twell_status s);

/*
 * Workspace bytes needed by twell_pack / twell_up_pack / twell_spmm /
 * twell_ffn_forward for these sizes (the maximum over the four calls).  gated is
 * 0 or 1.  Returns 0 for invalid shapes.  The workspace is scratch: its contents
 * need no initialisation and are undefined after a call.  For M > 256 and
 * d_model > 256 it includes 80 MiB of fp32 partial tiles used when the
 * tensor-core down-projection shares 128 x 512 tiles of y between SMs; for
 * 1 <= M <= 256 it includes a bitmap of d_ff / 32 + 1 words, the hidden units
 * that some token of the batch uses (the decode-size down-projection of up to
 * 32 tokens reads only those rows of W_down).
 */
size_t twell_workspace_bytes(int M, int d_model, int d_ff, int tile_w, int ell_w, int gated,
                             int ovf_capacity);

/*
 * twell_pack -- dense hidden activations h -> TwELL (+ dense backup).
 *   h      [M][ld_h] bf16 (ld_h >= d_ff, ld_h % 8 == 0); only columns < d_ff are read.
 *   out    fully described destination matrix (out->M, d_ff, tile_w, ell_w must
 *          equal the arguments).  Every field of *out is written.
 * The TwELL definition is the one above (upppp.jp 2026-05-11, TwELL section).
 */
twell_status twell_pack(const uint16_t *h, int M, int d_ff, int ld_h, int tile_w, int ell_w,
                        const twell_matrix *out, void *ws, size_t ws_bytes, void *stream);

/*
 * twell_up_pack -- the fused producer: z = x W_up^T (+ b), h = bf16(ReLU(z)),
 * or gated h = bf16(ReLU(x W_gate^T + b) * (x W_up^T)), written straight into
 * TwELL without a dense h in memory ("builds TwELL on the fly", upppp.jp
 * 2026-05-11, TwELL section).
 *   x       [M][d_model] bf16
 *   W_up    [d_ff][d_model] bf16 (row j = hidden unit j)
 *   W_gate  [d_ff][d_model] bf16 or NULL (non-gated)
 *   b       [d_ff] bf16 or NULL; with W_gate it is the gate bias
 *   z_debug NULL, or fp32 [M][d_ff] (non-gated: x W_up^T before the bias) /
 *           [M][2*d_ff] (gated: per row, d_ff gate values then d_ff up values).
 *           Test hook: lets a caller re-derive h exactly from the GPU's own fp32
 *           accumulators.
 * Gated requires tile_w <= 128.  ell_w <= 64 on this fused path.
 */
twell_status twell_up_pack(const uint16_t *x, const uint16_t *W_up, const uint16_t *W_gate,
                           const uint16_t *b, int M, int d_model, int d_ff, int tile_w,
                           int ell_w, const twell_matrix *out, float *z_debug, void *ws,
                           size_t ws_bytes, void *stream);

/*
 * twell_up_pack_stats -- twell_up_pack that also returns, per token, the
 * statistics an L1 activation regulariser works with (the pages pair ReLU
 * sparsity with an L1 penalty: upppp.jp 2026-05-11, sections
 * 「LLMフィードフォワード層の「無駄」とは何か」 and 「実際の性能改善」).  The sums are
 * taken in the producer's epilogue from the bf16 hidden values it packs.
 *   l1      [M] fp32 or NULL: sum over the token's hidden units of |h|.  fp32 sums
 *           in a fixed order (per tile in column order, then a fixed tree over
 *           tiles): the same on every run, within fp32 rounding of the exact sum.
 *   nnz_row [M] int32 or NULL: the token's number of nonzero h values.
 * Other arguments, the TwELL output and the limits as in twell_up_pack.  The
 * workspace (twell_workspace_bytes) holds the per-(token, tile) partial sums.
 */
twell_status twell_up_pack_stats(const uint16_t *x, const uint16_t *W_up, const uint16_t *W_gate,
                                 const uint16_t *b, int M, int d_model, int d_ff, int tile_w,
                                 int ell_w, const twell_matrix *out, float *l1, int32_t *nnz_row,
                                 void *ws, size_t ws_bytes, void *stream);

/*
 * twell_spmm -- y = h W_down reading h only from TwELL + backup.
 *   W_down [d_ff][d_model] bf16 (row j = hidden unit j's output vector)
 *   y      [M][d_model] bf16 (fp32 accumulation, one rounding at the end)
 *   mode   a twell_down_mode.
 * If the matrix's status word holds TWELL_ERR_OVERFLOW_CAPACITY, y is undefined.
 */
twell_status twell_spmm(const twell_matrix *a, const uint16_t *W_down, int d_model,
                        uint16_t *y, int mode, void *ws, size_t ws_bytes, void *stream);

/*
 * twell_ffn_forward -- the whole layer: twell_up_pack followed by twell_spmm on
 * the same stream.  `twell` receives the packed activations (it is the
 * intermediate, left populated).  Arguments as in the two calls above.
 */
twell_status twell_ffn_forward(const uint16_t *x, const uint16_t *W_up, const uint16_t *W_gate,
                               const uint16_t *b, const uint16_t *W_down, int M, int d_model,
                               int d_ff, int tile_w, int ell_w, const twell_matrix *twell,
                               uint16_t *y, int mode, void *ws, size_t ws_bytes, void *stream);

/*
 * twell_pack_noalloc -- twell_pack for callers that cannot provide a workspace.
 * The paper has no counterpart to this call; it exists for deployment.
 *
 * twell_pack needs caller-owned scratch.  Callers that cannot allocate device
 * memory when they pack -- a serving runtime that reserved the whole GPU up front
 * and forbids cudaMalloc on its request path, or a plugin interface that hands
 * over only input and output buffers -- use this variant instead.  It takes the
 * same arguments minus the workspace, produces the same output, and allocates
 * nothing: its scratch is a fixed 4 MiB device array inside the library, which
 * every GPU that loads the library holds until the process exits.
 *   - Scratch needed: 64 + 8*M + ovf_capacity*(4 + 2*tile_w) bytes, each part
 *     rounded up to 256.  A call needing more than 4 MiB returns
 *     TWELL_ERR_WORKSPACE without doing anything (e.g. M = 4096, tile_w = 128
 *     allows ovf_capacity up to about 15,900).
 *   - The first call on a device looks up the array's device address (once per
 *     device, with that device current).  Make that first call before any CUDA
 *     stream capture.  The address is kept for the life of the process and
 *     belongs to the device's primary context: do not call this entry point
 *     after cudaDeviceReset on that device, nor from a non-primary driver
 *     context.
 *   - Arguments are checked by the same code as twell_pack's, with the same
 *     results; M == 0 is a no-op that reads neither `h` nor `out`.
 *   - All calls share the one array and it keeps the previous call's contents;
 *     each call clears what must start at zero.  Calls whose executions overlap
 *     on the GPU (different streams, or different host threads, without ordering
 *     between them) race on the array and give undefined results.
 */
twell_status twell_pack_noalloc(const uint16_t *h, int M, int d_ff, int ld_h, int tile_w,
                                int ell_w, const twell_matrix *out, void *stream);

/*
 * twell_ffn_backward -- backward pass of the non-gated layer
 * y = bf16(ReLU(x W_up^T + b)) W_down through the forward's hybrid sparse form:
 * the pages' training kernel computes the whole backward pass without dense
 * matmuls on the sparse-main plus dense-backup representation (upppp.jp
 * 2026-05-11, section 「TwELLとカスタムCUDAカーネルが解決する課題」).
 *   h        the forward's TwELL of this layer (twell_up_pack / twell_ffn_forward on
 *            the same x), read only.  Its status word also receives this call's
 *            asynchronous errors (a bounded wait that gave up, capacity below).
 *   dY       [M][d_model] bf16: gradient of the loss with respect to y.
 *   dX       [M][d_model] bf16 out:   dZ W_up
 *   dW_up    [d_ff][d_model] bf16 out: dZ^T x
 *   db       [d_ff] fp32 out:          sum over tokens of dZ
 *   dW_down  [d_ff][d_model] bf16 out: h^T dY
 * where dZ = (dY W_down^T) masked to the entries h packs (the ReLU derivative is
 * taken as 1 where the stored h is nonzero), rounded once to bf16.  Products
 * accumulate in fp32 and round once.  h^T and dZ^T are packed internally as TwELL
 * with tiles of 128 tokens, ell_w_t slots and ovf_capacity_t backup rows (a
 * smaller capacity than the pairs that overflow raises TWELL_ERR_OVERFLOW_CAPACITY
 * in h's status word and leaves the weight gradients undefined).
 * Limits: M and d_ff multiples of 128, tile_w <= 128, 1 <= ell_w_t <= 128,
 * d_model % 64 == 0.  Workspace: twell_backward_workspace_bytes.
 */
size_t twell_backward_workspace_bytes(int M, int d_model, int d_ff, int tile_w, int ell_w,
                                      int ovf_capacity, int ell_w_t, int ovf_capacity_t);
twell_status twell_ffn_backward(const uint16_t *x, const uint16_t *W_up, const uint16_t *W_down,
                                const twell_matrix *h, const uint16_t *dY, int d_model, int ell_w_t,
                                int ovf_capacity_t, uint16_t *dX, uint16_t *dW_up, float *db,
                                uint16_t *dW_down, void *ws, size_t ws_bytes, void *stream);

/*
 * twell_spmm_token_overflow -- y = h W_down with the backup read the other way
 * (the whole-token reading of "rows that overflow spill to a dense backup"): a
 * token with any tile holding more than ell_w nonzeros is taken out of the ELL
 * form and its whole hidden row is stored fully dense (as TwELL with
 * ell_w = tile_w) and run as a small dense product; the other tokens use their
 * ELL slots.  Built from the per-(token, tile) form `a` so the two readings can
 * be compared on the same data (backup size, time).
 *   cap_tok  rows available for overflowing tokens; more sets
 *            TWELL_ERR_OVERFLOW_CAPACITY in a's status word (y undefined).
 *   n_tok    device int32 or NULL: number of overflowing tokens.
 * Other arguments as twell_spmm (AUTO down-path selection).  Workspace:
 * twell_token_overflow_workspace_bytes.
 */
size_t twell_token_overflow_workspace_bytes(int M, int d_model, int d_ff, int tile_w, int ell_w,
                                            int cap_tok);
twell_status twell_spmm_token_overflow(const twell_matrix *a, const uint16_t *W_down, int d_model,
                                       uint16_t *y, int cap_tok, int32_t *n_tok, void *ws,
                                       size_t ws_bytes, void *stream);

/*
 * twell_down_schedule -- diagnostic, host only (no GPU, nothing launched): the
 * work split of the token-major tensor-core down-projection (twell_spmm, MMA
 * path, M > 256) for these sizes on a GPU with num_sms SMs, from the same
 * planning and scheduling code the kernel runs.  Writes at most out_len int32
 * to out (host memory, may be NULL) and returns the number needed, or -1 for
 * shapes that do not take this kernel.  Layout: a header
 *   [split (0 whole tiles, 1 split-K, 2 even deal of K chunks), CTAs, tiles, K steps]
 * then, per CTA in order and per segment in its order, 7 values
 *   [cta, tile, first K step, end K step, CTAs sharing the tile (1: whole tile),
 *    arrival counter index (-1), partial-tile slot (-1)].
 * Tiles are 128 tokens x 512 columns of y (256 when d_model <= 256).  The paper
 * has no counterpart.
 */
int twell_down_schedule(int M, int d_model, int d_ff, int tile_w, int ell_w, int num_sms, int32_t *out,
                        int out_len);

/*
 * twell_selftest_bounded_wait -- diagnostic for the failure path.  Every wait of
 * the tensor-core kernels on a shared-memory barrier is bounded (about 2 s of
 * device wall clock); one that gives up records TWELL_ERR_TIMEOUT and the kernel
 * unwinds.  This call runs that same wait on a barrier that nothing arrives on:
 * it must give up, set *status (device int32, caller-initialised to 0) to
 * TWELL_ERR_TIMEOUT and write the wait's duration in ns to *elapsed_ns (device
 * u64).  Asynchronous; the kernel takes about 2 s.  The paper has no counterpart.
 */
twell_status twell_selftest_bounded_wait(int32_t *status, unsigned long long *elapsed_ns,
                                         void *stream);

/*
 * Synchronise `stream`, then return the matrix's device status word (TWELL_OK if
 * clean) and, if n_ovf_out is not NULL, the true overflow-pair count.
 */
twell_status twell_read_status(const twell_matrix *a, void *stream, int32_t *n_ovf_out);

#ifdef __cplusplus
}
#endif
#endif /* TWELL_B200_H */
