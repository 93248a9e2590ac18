/*
 * fa.h -- C ABI of libfa.so: exact softmax attention forward on B200 (sm_100a).
 *
 * The operation is the dense attention definition O = softmax(Q K^T / sqrt(d)) V
 * (lihaoran.work, "FlashAttention: the intermediate matrix comes first", the
 * opening formula), computed in one fused pass that keeps per-row running
 * statistics -- the maximum m, the denominator l and the unnormalised
 * numerator u -- and rescales them whenever a later key tile raises the
 * maximum (liminalml.com "FlashAttention", the block update and "output u/l"
 * after the final block; interactiveml.org "FlashAttention saves the matrix,
 * not the quadratic work", the three sufficient statistics).  The N x N score
 * matrix never reaches global memory (sadullah.online "Flash Attention
 * Explained", fused tiled computation).
 *
 * Conventions shared by every entry point:
 *   - Tensors are dense, row-major, in device memory owned by the caller:
 *       Q, K, V, O : bfloat16 [B][H][N][d]   (d fastest)
 *       LSE        : float32  [B][H][N]
 *   - Calls are asynchronous on the given stream (a cudaStream_t passed as
 *     void*; NULL = the legacy default stream).  Nothing is valid until the
 *     stream has been synchronised.
 *   - The library never allocates device memory.
 *   - Errors are returned as fa_status; argument errors are reported before
 *     anything is launched.  Device-side failures (a bounded wait that gave
 *     up) are reported by fa_get_device_status().
 */
#ifndef FA_H_
#define FA_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum fa_status {
  FA_OK = 0,
  FA_ERR_NULL = 1,            /* a required pointer is NULL                       */
  FA_ERR_SHAPE = 2,           /* B, H or N < 1, sizes overflow, or scale not finite */
  FA_ERR_UNSUPPORTED = 3,     /* d not in {64, 128}, scale <= 0, or not an sm_100 GPU */
  FA_ERR_ALIGN = 4,           /* a pointer is not 16-byte aligned (LSE: 4-byte)   */
  FA_ERR_CUDA = 5,            /* a CUDA runtime/driver call or the launch failed  */
  FA_ERR_DEVICE_TIMEOUT = 6,  /* a kernel gave up on a bounded wait               */
  FA_ERR_ALIAS = 7,           /* O, LSE or a workspace overlaps another argument  */
  FA_ERR_WORKSPACE = 8,       /* the workspace is smaller than required           */
  FA_ERR_LAYOUT = 9,          /* a block-sparse list was out of range or order    */
  FA_ERR_BOUNDS = 10          /* an index check of the debug build failed          */
} fa_status;

/*
 * fa_fwd -- O = softmax(scale * Q K^T [+ causal mask]) V, and its log-sum-exp.
 *
 *   Q, K, V  device, bf16 [B][H][N][d], read only; they may alias each other.
 *   O        device, bf16 [B][H][N][d], written:
 *              O[b,h,i,:] = sum_j w_ij V[b,h,j,:] / sum_j w_ij,
 *              w_ij = exp(scale * <Q[b,h,i,:], K[b,h,j,:]> - m_i)
 *            over the allowed keys j (all j, or j <= i when causal != 0),
 *            rounded to bf16 (round to nearest even).
 *   LSE      device, fp32 [B][H][N], written: ln sum_j exp(scale * <q_i, k_j>)
 *            over the allowed keys (natural log of the scaled scores).  May be
 *            NULL, in which case it is not written.
 *   B, H, N  batch, heads, sequence length (queries and keys), each >= 1;
 *            any N is accepted (ragged last tile is masked).
 *   d        head width: 64 or 128.
 *   scale    positive finite multiplier of the dot product (1/sqrt(d) for the
 *            standard definition).
 *   causal   0: every key is allowed; nonzero: query i sees keys j <= i.
 *   stream   cudaStream_t (as void*) on which the kernel is launched.
 *
 * Q, K, V and O must be 16-byte aligned; LSE 4-byte aligned.  O and LSE must
 * not overlap the inputs or each other.  Returns FA_OK once the kernel is
 * enqueued.
 */
fa_status fa_fwd(const void* Q, const void* K, const void* V, void* O, float* LSE, int B, int H,
                 int N, int d, float scale, int causal, void* stream);

/*
 * fa_fwd_splitkv -- the same result as fa_fwd, with the key range of every
 * query block divided into num_splits ranges processed as separate work items, for
 * problems with too few query blocks to fill the GPU.  Each range leaves a
 * partial state -- its normalised output u/l and its log-sum-exp -- and a
 * second kernel merges the states of a row: with M = max_s LSE_s and
 * w_s = e^(LSE_s - M) (0 for a range with no allowed key), O = sum w_s O_s /
 * sum w_s and LSE = M + ln sum w_s.  This is the block update of liminalml.com
 * "FlashAttention" (rescale both numerator and denominator by e^(m - m')) and
 * the block merge of interactiveml.org (old scale 0 while m = -inf), applied
 * to whole partial states.
 *
 *   Q, K, V, O, LSE, B, H, N, d, scale, causal, stream: as for fa_fwd.
 *   workspace        device memory owned by the caller, 16-byte aligned, at
 *                    least fa_fwd_splitkv_workspace_bytes(B, H, N, d,
 *                    causal, num_splits) bytes; overwritten (fp32 partial outputs
 *                    [splits][B*H*N][d] followed by partial LSE
 *                    [splits][B*H*N], splits = the ranges that remain, below);
 *                    must not overlap any other argument.  When one range
 *                    remains it is not used at all and may be NULL.
 *   workspace_bytes  its size.
 *   num_splits       1..256; <= 0 picks fa_fwd_splitkv_default_splits().
 *                    Ranges are ceil(ceil(N/128) / num_splits) key tiles;
 *                    trailing empty ranges are dropped.  When one range
 *                    remains, the fused kernel of fa_fwd runs alone.
 * Errors as fa_fwd, plus (only when more than one range remains) FA_ERR_NULL
 * for a NULL workspace, FA_ERR_ALIGN for a misaligned one, FA_ERR_WORKSPACE
 * when it is too small; FA_ERR_UNSUPPORTED for num_splits > 256.  Two kernels
 * are enqueued on `stream` (one when a single range remains).
 */
fa_status fa_fwd_splitkv(const void* Q, const void* K, const void* V, void* O, float* LSE,
                         void* workspace, size_t workspace_bytes, int B, int H, int N, int d,
                         float scale, int causal, int num_splits, void* stream);

/* Bytes of workspace fa_fwd_splitkv needs for the ranges that remain after
 * empty ones are dropped: 0 when a single range remains (no workspace is
 * used) and 0 for invalid arguments.  num_splits <= 0 means the default for
 * this shape and mask. */
size_t fa_fwd_splitkv_workspace_bytes(int B, int H, int N, int d, int causal, int num_splits);

/* Default split count: non-causal, the most ranges that fit in one wave of
 * 148 SMs; causal, at least 1.5 waves; at least two key tiles per range
 * (1 for invalid arguments). */
int fa_fwd_splitkv_default_splits(int B, int H, int N, int d, int causal);

/*
 * fa_bwd -- gradients of L = sum(O * dO) for O = fa_fwd(Q, K, V): dQ, dK, dV,
 * recomputing the probabilities tile by tile from Q, K and the forward's LSE
 * (lihaoran.work, "selected recomputation in the backward pass"; the
 * derivative of the definition: dV = P^T dO, dS = P * (dO V^T - D) with
 * D = rowsum(dO * O), dQ = scale dS K, dK = scale dS^T Q).
 *
 *   Q, K, V, O, dO  device, bf16 [B][H][N][d], read (O as written by fa_fwd).
 *   LSE             device, fp32 [B][H][N], read (as written by fa_fwd with the
 *                   same scale and mask: finite for every row).
 *   dQ, dK, dV      device, bf16 [B][H][N][d], written.
 *   workspace       device, 16-byte aligned, >= fa_bwd_workspace_bytes(B, H,
 *                   N) bytes, overwritten: LSE * log2(e) and D, each fp32
 *                   [B][H][N rounded up to 128], then the fp32 accumulator
 *                   of dS K, [B][H][N rounded up to 128][d].
 *   B, H, N, d, scale, causal, stream: as for fa_fwd.
 * The outputs and the workspace must not overlap the inputs or each other.
 * Three kernels are enqueued on `stream`: the row dots (and the accumulator
 * cleared), dK and dV with every key tile's share of dQ added into the
 * accumulator (fp32 reductions at L2, so dQ's rounding depends on the order
 * in which they land: results may differ from run to run in the last bits),
 * and dQ converted to bf16.  Errors as fa_fwd, plus FA_ERR_WORKSPACE for a
 * short workspace; device-side give-ups are reported by
 * fa_get_device_status().
 */
fa_status fa_bwd(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                 const float* LSE, void* dQ, void* dK, void* dV, void* workspace,
                 size_t workspace_bytes, int B, int H, int N, int d, float scale, int causal,
                 void* stream);

/* Bytes of workspace fa_bwd needs: (2 + 128) * 4 * B * H * (N rounded up to
 * 128), enough for either head dimension; 0 for invalid arguments. */
size_t fa_bwd_workspace_bytes(int B, int H, int N);

/* Size of the workspace built into the library for fa_fwd_splitkv_noalloc. */
#define FA_NOALLOC_SCRATCH_BYTES (64 * 1024 * 1024)

/*
 * fa_fwd_splitkv_noalloc -- fa_fwd_splitkv for callers that cannot allocate
 * device memory when they run attention: code being captured into a CUDA
 * graph that must not gain allocation nodes, runtimes that forbid allocation
 * after start-up, or programs whose device memory belongs to another
 * framework's pool.  The pages describe no such entry point; it has no
 * counterpart there.
 *
 * Instead of a caller's workspace it uses an array of
 * FA_NOALLOC_SCRATCH_BYTES (64 MiB) that is part of this library's device
 * code: every GPU that loads the library holds that memory until the process
 * exits.  The caller still passes Q, K, V, O and LSE, with the meaning,
 * layout and errors of fa_fwd_splitkv (num_splits <= 0 picks the default).
 *
 *   - A problem whose workspace (fa_fwd_splitkv_workspace_bytes, counted
 *     for the ranges that remain) exceeds FA_NOALLOC_SCRATCH_BYTES is
 *     rejected with FA_ERR_WORKSPACE before anything is enqueued.  A problem
 *     that runs as a single range needs none and is never rejected for size.
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current) and keeps it; make
 *     that first call before any stream capture.  The library allocates
 *     nothing, on any call.
 *   - All calls on a device share the one array, which keeps whatever the
 *     last call left in it (nothing in it needs to start at zero).  Calls
 *     that may overlap on the GPU -- on different streams without ordering,
 *     or from several host threads -- race on it and must be serialised by
 *     the caller.
 *   - After fa_get_device_status() reports FA_ERR_DEVICE_TIMEOUT for such a
 *     call, O and LSE are undefined and may hold values merged from partial
 *     states an earlier call left in the array.
 */
fa_status fa_fwd_splitkv_noalloc(const void* Q, const void* K, const void* V, void* O, float* LSE,
                                 int B, int H, int N, int d, float scale, int causal, int num_splits,
                                 void* stream);

/*
 * fa_fwd_tile_config -- fa_fwd with a chosen tile shape, for measuring how
 * wall-clock time depends on the tile size (interactiveml.org
 * "FlashAttention saves the matrix, not the quadratic work", the suggested
 * experiments: vary tile size and head width).
 *   query_rows  query rows per work item: 256 (two 128-row tiles whose softmax and
 *               MMAs ping-pong, as fa_fwd) or 128 (one tile, no ping-pong);
 *               0 = 256.
 *   key_tile    keys per score tile: 128 (as fa_fwd) or 64; 0 = 128.
 * The query tile itself is always 128 rows: the tensor core's M.  (256, 128)
 * is fa_fwd; the other shapes run the same kernel template and agree with it
 * to rounding.  Arguments and errors as fa_fwd, plus FA_ERR_UNSUPPORTED for
 * any other shape.
 */
fa_status fa_fwd_tile_config(const void* Q, const void* K, const void* V, void* O, float* LSE, int B,
                             int H, int N, int d, float scale, int causal, int query_rows, int key_tile,
                             void* stream);

/*
 * fa_fwd_host -- fa_fwd on inputs and outputs in HOST memory: the end-to-end
 * call.  Q, K, V are copied to the device, the forward runs there, and O and
 * LSE are copied back, all pipelined over `chunks` groups of heads on three
 * streams of the library's own.  While one group is copied in, the previous
 * one is computed and the one before is copied out.  Each (b, h) pair needs
 * only its own Q, K, V (lihaoran.work, the opening formula), so the split
 * does not change any output bit.
 *
 *   Qh, Kh, Vh   host, bf16 [B][H][N][d], read.  Pinned memory
 *                (cudaHostAlloc / cudaHostRegister) lets the copies overlap;
 *                pageable memory works but serialises them.
 *   Oh           host, bf16 [B][H][N][d], written.
 *   LSEh         host, fp32 [B][H][N], written; may be NULL.
 *   workspace    device, 16-byte aligned, >= fa_fwd_host_workspace_bytes(B,
 *                H, N, d) bytes: the device copies of Q, K, V, O, LSE.
 *   chunks       groups of heads (<= 0: 8; capped at B*H and 64).
 *   B, H, N, d, scale, causal: as fa_fwd.
 *   stream       the caller's stream: the work starts after what is already
 *                queued on it, and work queued on it afterwards waits until
 *                O and LSE have reached host memory.  Synchronise it before
 *                reading them.
 * The first call on a device creates the library's three streams and its
 * events (no device memory).  Calls from several host threads are enqueued
 * one at a time; their work shares the three streams.  Errors: as fa_fwd, plus FA_ERR_WORKSPACE for a
 * short workspace and FA_ERR_UNSUPPORTED when a host argument is device or
 * managed memory or the workspace is not device memory.
 */
fa_status fa_fwd_host(const void* Qh, const void* Kh, const void* Vh, void* Oh, float* LSEh,
                      void* workspace, size_t workspace_bytes, int B, int H, int N, int d, float scale,
                      int causal, int chunks, void* stream);

/* Device workspace bytes fa_fwd_host needs: 8*B*H*N*d + 4*B*H*N (0 if invalid). */
size_t fa_fwd_host_workspace_bytes(int B, int H, int N, int d);

/* Block of the block-sparse layout: query rows x keys. */
#define FA_BLOCK_Q 256
#define FA_BLOCK_K 128

/*
 * fa_fwd_block_sparse -- attention over the key blocks a block layout
 * retains: query i sees key j only if j's key block is in the list of i's
 * query block (and j <= i when causal != 0).  The pages call sparsity a
 * separate design dimension, choosing which query-key interactions are kept
 * (liminalml.com "FlashAttention", "Is it sparse attention?"), and suggest
 * comparing exact and block-sparse attention at matched output error
 * (interactiveml.org "FlashAttention saves the matrix, not the quadratic
 * work", the suggested experiments).  Over the retained keys the result is
 * the exact softmax, computed as in fa_fwd; with every block retained it is
 * fa_fwd's result, bit for bit.
 *
 *   Q, K, V, O, LSE, B, H, N, d, scale, causal, stream: as in fa_fwd.
 *   block_row_ptr  device, int32 [ceil(N / FA_BLOCK_Q) + 1], read: query
 *                  block r (rows FA_BLOCK_Q*r ...) retains the key blocks
 *                  block_col_idx[block_row_ptr[r] .. block_row_ptr[r+1]-1].
 *   block_col_idx  device, int32 [nnz], read: key block numbers (keys
 *                  FA_BLOCK_K*c ...), strictly ascending within each query
 *                  block, each in [0, ceil(N / FA_BLOCK_K)).  May be NULL when
 *                  nnz == 0.
 *   nnz            entries of block_col_idx (>= 0).
 * One layout serves every (b, h).  A query with no retained key gets O = 0
 * and LSE = -inf.  Key blocks past a causal block's last row are skipped.
 *
 * Errors: as fa_fwd, plus FA_ERR_NULL (no block_row_ptr, or no block_col_idx
 * with nnz > 0), FA_ERR_SHAPE (nnz < 0), FA_ERR_ALIGN (a list not 4-byte
 * aligned), FA_ERR_ALIAS (O or LSE overlaps a list).  The lists live on the
 * device and are checked there: an entry out of range or out of order is
 * masked out (nothing outside the tensors is read), the outputs are then
 * undefined, and fa_get_device_status() reports FA_ERR_LAYOUT.
 */
fa_status fa_fwd_block_sparse(const void* Q, const void* K, const void* V, void* O, float* LSE,
                              const int* block_row_ptr, const int* block_col_idx, int nnz, int B,
                              int H, int N, int d, float scale, int causal, void* stream);

/*
 * fa_softmax_rows -- the softmax step of standard (materialising) attention,
 * kept as a comparator: standard attention writes the N x N scores to
 * global memory, reads them back for the softmax, writes the probabilities
 * and reads them again for the product with V (sadullah.online "Flash
 * Attention Explained", the memory-movement section; interactiveml.org, the
 * square table of scores written to and read back from HBM).
 *
 *   S    device, fp32 [BH][N][N], read: the raw dot products q_i . k_j.
 *   P    device, bf16 [BH][N][N], written: softmax_j(scale * S[i][j]) over the
 *        allowed keys (j <= i when causal), 0 elsewhere.
 *   LSE  device, fp32 [BH][N], written (may be NULL): ln sum_j e^(scale S_ij).
 *   N    must be even (rows of P stay 4-byte aligned); scale > 0.
 * Asynchronous on `stream`.  FA_ERR_NULL / _SHAPE / _UNSUPPORTED / _ALIGN
 * for bad arguments, FA_ERR_CUDA if the launch fails.
 */
fa_status fa_softmax_rows(const float* S, void* P, float* LSE, int BH, int N, float scale,
                          int causal, void* stream);

/* Human-readable name of a status code (static string, never NULL). */
const char* fa_status_string(fa_status status);

/*
 * fa_get_device_status -- synchronise `stream`, then read and clear the
 * device status words (forward and backward kernels) of the current device.
 * Returns FA_ERR_DEVICE_TIMEOUT
 * if any kernel launched by this library gave up on a bounded wait since the
 * last call (its outputs are then undefined), FA_ERR_BOUNDS if, in a library
 * built with -DFA_DEBUG, an index check failed (the access was skipped and
 * the outputs are undefined), FA_ERR_LAYOUT if a block-sparse call met a
 * malformed list (and nothing else failed), FA_ERR_CUDA if the
 * synchronisation failed, FA_OK otherwise.
 */
fa_status fa_get_device_status(void* stream);

/*
 * fa_get_device_status_word -- as fa_get_device_status, and also stores the
 * raw status word in *word (0 = no failure; bit 0 = a wait gave up; bit 1 = a
 * malformed block-sparse list; bit 2 = an index check of a debug build
 * failed; bit 8+k = the wait at site k gave up; bit 16+k = the index check
 * at site k failed, for diagnosis).  word may be NULL.
 */
fa_status fa_get_device_status_word(void* stream, unsigned int* word);

/* Message of the last CUDA error seen by this library in the calling thread
 * ("" if none).  Static thread-local storage; valid until the next call. */
const char* fa_last_cuda_error(void);

/*
 * fa_set_debug -- test hook.  Applies to kernels launched afterwards from any
 * thread.  timeout_ns: how long a bounded wait inside a kernel may spin
 * before it gives up (0 = default, 2 s).  flags bit 0: make the softmax
 * warps of every CTA wait on a barrier that nothing arrives at, so that the
 * wait runs out, the CTA unwinds without trapping, and
 * fa_get_device_status() reports FA_ERR_DEVICE_TIMEOUT.  flags = 0 restores
 * normal operation.
 */
void fa_set_debug(unsigned int flags, unsigned long long timeout_ns);

/* Library version as "major.minor.patch" (static string). */
const char* fa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FA_H_ */
