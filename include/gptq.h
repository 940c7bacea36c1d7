/*
 * gptq.h — C ABI of libgptq.so, a B200 (sm_100a) GPTQ layer-wise quantization solver.
 *
 * The calls follow the per-layer flow of "GPTQ量化算法深度解析：从Hessian曲率到大模型单卡部署"
 * (sheratonhq.com) §3.1: add calibration batches to the Hessian (step 1), factor it
 * (step 2), sweep the columns in blocks with error feedback (step 3), store codes and
 * quantization parameters (step 4).  Quantizer parameters (bits, group size, sym,
 * desc_act, damp_percent) are those of §3.3 of the same page and of the table
 * "bits、group_size、sym 与 desc_act 分别影响什么" of the lansai.wang deployment guide.
 *
 * Conventions shared by every call
 *  - Array arguments are DEVICE pointers owned by the caller; the library never
 *    allocates or frees device memory.  Scratch memory is the caller's `ws`
 *    buffer, sized with gptq_workspace_size().
 *  - Every call is asynchronous on `stream` (a cudaStream_t passed as void*;
 *    NULL = the legacy default stream).  Host-side results (n_seen) are updated
 *    at enqueue time.
 *  - Return value: GPTQ_OK, or exactly one error code.  Argument errors are
 *    detected on the host before anything is launched.  GPTQ_ERR_CUDA means a
 *    launch failed (cudaGetLastError() was not cudaSuccess).
 *  - Conditions only the device can see are OR-ed as gptq_status bits into
 *    `*dev_status` (a caller-owned device int32, may be NULL to ignore them):
 *    GPTQ_ERR_NOT_PD (non-positive pivot), GPTQ_ERR_NONFINITE (NaN/Inf in H),
 *    GPTQ_ERR_INVALID_ARG (a caller-supplied permutation is not a permutation),
 *    GPTQ_ERR_TIMEOUT (a bounded device wait gave up).  Kernels never trap; the
 *    caller reads *dev_status after synchronizing the stream.
 *  - Matrices are row-major.  W is rows x cols (out x in features, as a PyTorch
 *    Linear weight); X is tokens x cols.
 *  - Host threads: the calls may be made from several host threads at once.  The
 *    side stream of gptq_quantize_layer and the text of gptq_last_error are kept
 *    per host thread, and the launch counter is atomic; gptq_prepare_static is the
 *    one call whose scratch memory is shared (see there).
 */
#ifndef GPTQ_H_
#define GPTQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes.  Values are distinct bits so device conditions can be OR-ed. */
typedef enum {
  GPTQ_OK = 0,
  GPTQ_ERR_INVALID_ARG = 1,
  GPTQ_ERR_UNSUPPORTED = 2,
  GPTQ_ERR_WORKSPACE = 4,
  GPTQ_ERR_NOT_PD = 8,
  GPTQ_ERR_NONFINITE = 16,
  GPTQ_ERR_TIMEOUT = 32,
  GPTQ_ERR_CUDA = 64
} gptq_status;

/* Element types of W and X. */
typedef enum { GPTQ_F32 = 0, GPTQ_F16 = 1, GPTQ_BF16 = 2 } gptq_dtype;

/* act_order values. */
enum { GPTQ_ORDER_NATURAL = 0, GPTQ_ORDER_DESC_DIAG = 1, GPTQ_ORDER_GIVEN = 2 };

/* Workspace queries. */
enum { GPTQ_OP_PREPARE = 1, GPTQ_OP_QUANTIZE = 2 };

/*
 * Quantizer configuration (GPTQ量化算法深度解析 §3.3; lansai.wang guide, parameter table).
 *  bits        2, 3, 4 or 8: codes take values 0 .. 2^bits - 1.
 *  group_size  0 (or -1): one grid per row, from the row before any compensation.
 *              g > 0: one grid per g consecutive columns in sweep order, computed when
 *              the sweep reaches the group's first column from the current compensated
 *              weights.  g must divide 128 (the kernels' column panel).
 *  sym         0: asymmetric min-max grid containing 0, integer zero-point
 *              z = rint(-lo/s).  1: symmetric range [-max|v|, max|v|], z = 2^(bits-1).
 *  act_order   GPTQ_ORDER_NATURAL, GPTQ_ORDER_DESC_DIAG (columns by descending
 *              diag(H), ties by ascending index; "desc_act"), or GPTQ_ORDER_GIVEN
 *              (perm supplied by the caller to gptq_prepare).
 *  damp        relative damping: lambda = damp * mean(diag H) is added to diag H.
 *  block_size  lazy-batch width B of §2.4.  Lazy batching is exact, so B changes
 *              rounding only; the kernels always sweep 128-column panels.  Must be
 *              >= 1, and group_size must divide B or be a multiple of it.
 */
typedef struct {
  int bits;
  int group_size;
  int sym;
  int act_order;
  float damp;
  int block_size;
} gptq_config;

/*
 * gptq_workspace_size — bytes of `ws` needed by gptq_prepare (op = GPTQ_OP_PREPARE)
 * or gptq_quantize_layer (op = GPTQ_OP_QUANTIZE) for the given shape.  Returns 0
 * for invalid arguments.  The result is a multiple of 256.
 */
size_t gptq_workspace_size(int op, int64_t rows, int64_t cols, const gptq_config* cfg);

/*
 * gptq_hessian_accumulate — GPTQ量化算法深度解析 §3.1 step 1 (H = 2 X X^T, normalised).
 * Adds a chunk of m calibration tokens to the running Hessian:
 *     H <- H * n/(n+m) + (2/(n+m)) * X^T X,      n <- n + m
 *  H        cols x cols fp32, row-major.  Only the upper triangle (i <= j) is read
 *           and written; the strictly lower triangle is left untouched.  When
 *           *n_seen == 0 the upper triangle is overwritten (need not be initialised).
 *  n_seen   HOST pointer to the number of tokens already in H; updated on enqueue.
 *  X        device pointer, m_tokens x cols, row stride ldx elements (ldx >= cols),
 *           element type xdtype.  16-bit X with ldx a multiple of 8 and a 16-byte
 *           aligned base runs on the tcgen05 tensor cores (fp32 accumulate).
 *  dev_status  see conventions (may be NULL).
 *  m_tokens == 0 is a no-op.  Errors: INVALID_ARG (null pointer, cols <= 0,
 *  m_tokens < 0, ldx < cols, bad dtype).
 */
gptq_status gptq_hessian_accumulate(float* H, int64_t* n_seen, const void* X, int xdtype,
                                    int64_t m_tokens, int64_t cols, int64_t ldx,
                                    int32_t* dev_status, void* stream);

/*
 * gptq_prepare — GPTQ量化算法深度解析 §3.1 step 2 and §2.4 (Cholesky), §3.3 (damping,
 * desc_act).  Reads the upper triangle of H, damps it by lambda = damp*mean(diag H),
 * orders the columns, and writes the inverse Cholesky factor of the permuted matrix:
 *     Hp = (H + lambda I)[perm][:, perm],     U upper triangular, U^T U = Hp^-1,
 *     U[q][q] > 0, entries below the diagonal written as 0.
 *  H     cols x cols fp32 (upper triangle used; not modified).
 *  U     cols x cols fp32 output, row-major.
 *  perm  cols int32: output for NATURAL / DESC_DIAG (perm[j] = original column
 *        swept j-th); input for GIVEN (checked on the device: a bad permutation
 *        sets GPTQ_ERR_INVALID_ARG in *dev_status).
 *  ws    workspace of at least gptq_workspace_size(GPTQ_OP_PREPARE, 0, cols, cfg)
 *        bytes, 256-byte aligned.
 *  Device conditions: NONFINITE (diag(H) not finite), NOT_PD (a pivot <= 0; the
 *  factor is then not meaningful).  Errors: INVALID_ARG, WORKSPACE.
 */
gptq_status gptq_prepare(const float* H, int64_t cols, const gptq_config* cfg, float* U,
                         int32_t* perm, void* ws, size_t ws_bytes, int32_t* dev_status,
                         void* stream);

/*
 * gptq_quantize_layer — GPTQ量化算法深度解析 §2.2 (OBS compensation), §2.4 (fixed order,
 * lazy batch updates), §3.1 step 3-4.  Sweeps the columns of W in the order perm,
 * 128 at a time.  For each column q (in sweep order), with d = U[q][q]:
 *     code = clamp(rint(w/s) + z, 0, 2^bits-1),  Q = s (code - z),
 *     err = (w - Q)/d,   w[q+1 : block end] -= err * U[q][q+1 : block end]
 * and after each block  W[:, end:] -= Err * U[block, end:].
 *  W       rows x cols, row stride ldw elements, element type wdtype; not modified.
 *  U, perm as produced by gptq_prepare.
 *  codes   rows x cols uint8, ORIGINAL column order.
 *  scales, zeros  rows x G fp32, G = ceil(cols/group_size) (1 for per-row grids),
 *          groups in sweep order; zeros hold integers.
 *  g_idx   cols int32: group of each original column (0 for per-row grids).
 *  losses  cols fp32: sum over rows of (w - Q)^2 / (2 d^2), ORIGINAL column order.
 *  ws      at least gptq_workspace_size(GPTQ_OP_QUANTIZE, rows, cols, cfg) bytes.
 *  rows == 0 writes only g_idx and zero losses.  Errors: INVALID_ARG,
 *  UNSUPPORTED (group_size does not divide 128, or not compatible with block_size),
 *  WORKSPACE.
 *  Streams: part of the lazy update runs on a library-owned side stream (one per
 *  host thread and device) that forks from `stream` at the start of the call and
 *  joins it before the call returns, through events; work enqueued on `stream`
 *  afterwards sees the complete result.  (Graph capture of this call has not been
 *  tested.)  The per-block update order is fixed, so the outputs are
 *  deterministic for a given U and W.
 */
gptq_status gptq_quantize_layer(const void* W, int wdtype, int64_t rows, int64_t cols,
                                int64_t ldw, const float* U, const int32_t* perm,
                                const gptq_config* cfg, uint8_t* codes, float* scales,
                                float* zeros, int32_t* g_idx, float* losses, void* ws,
                                size_t ws_bytes, int32_t* dev_status, void* stream);

/*
 * gptq_pack — packing of low-bit codes into integer words (gptq-for-llama article,
 * ainews.cool, "工程细节": four 4-bit codes per 16-bit integer).  Each row's codes
 * form a little-endian, LSB-first bitstream of `bits`-bit fields:
 *     code c occupies bits [c*bits, (c+1)*bits) of the row's stream,
 * stored as rows x ceil(cols*bits/32) uint32 words; trailing bits are zero.  Codes
 * are masked to `bits` bits.  bits in {2, 3, 4, 8}.  Errors: INVALID_ARG.
 */
gptq_status gptq_pack(const uint8_t* codes, int64_t rows, int64_t cols, int bits,
                      uint32_t* packed, void* stream);

/*
 * gptq_prepare_static — gptq_prepare for callers that cannot allocate device memory.
 * The GPTQ pages have no counterpart to this call; it exists for callers that cannot
 * allocate where they call us (a plugin inside a framework whose caching allocator
 * already holds the device memory, code given a fixed memory budget, a service that
 * must not allocate after start-up because allocation can block and synchronize).
 * Same arguments, results and device conditions as gptq_prepare, but no `ws`: the
 * scratch memory is an array of GPTQ_STATIC_SCRATCH_BYTES compiled into the library,
 * which every GPU that loads the library holds until the process exits.  The call
 * itself allocates nothing (no cudaMalloc, no cudaFree, no allocating library call).
 *  - cols > GPTQ_STATIC_MAX_COLS returns GPTQ_ERR_WORKSPACE before anything runs;
 *    use gptq_prepare with a caller workspace for larger layers.
 *  - The first call in a device's context looks up the array's device address
 *    (cudaGetSymbolAddress) with that device current and caches it with the
 *    context's id; make that first call before any stream capture.  After a
 *    device reset (a new context) the next call looks the address up again.
 *  - Every call shares the one array, which keeps the previous call's contents (the
 *    call clears what must start at zero itself).  Calls whose work overlaps on the
 *    GPU — e.g. on two streams at once — race on the array; order them on one stream
 *    or synchronize between them.
 */
#define GPTQ_STATIC_MAX_COLS 1024
#define GPTQ_STATIC_SCRATCH_BYTES (12u * 1024u * 1024u)
gptq_status gptq_prepare_static(const float* H, int64_t cols, const gptq_config* cfg, float* U,
                                int32_t* perm, int32_t* dev_status, void* stream);

/*
 * gptq_repack_sweep_order — the packed codes of gptq_pack (original column order)
 * rewritten in sweep order for gptq_dequant_matmul: column j of an output row holds
 * original column perm[j] (perm from gptq_prepare; NULL = identity).  Under
 * act-order a group's columns are scattered over the original order (the gather
 * desc_act costs at inference, GPTQ量化算法深度解析 §3.3); in sweep order every group
 * is one contiguous run and the gather moves to the small activation block.
 *  packed  rows x ceil(cols*bits/32) uint32 (gptq_pack layout)
 *  out     rows x (cols/32)*bits uint32, same bitstream layout, sweep order
 *  cols % 32 == 0, bits in {2,3,4,8}.  Errors: INVALID_ARG.
 */
gptq_status gptq_repack_sweep_order(const uint32_t* packed, int64_t rows, int64_t cols,
                                    int bits, const int32_t* perm, uint32_t* out,
                                    void* stream);
/*
 * gptq_dequant_matmul — Y = X Q^T from the stored form, decode-sized token counts
 * (gptq-for-llama article, "工程细节": products straight from packed 4-bit codes):
 *     Q[r][c] = scales[r][g(c)] (code[r][c] - zeros[r][g(c)])
 *  X       m_tokens x cols, row stride ldx, xdtype, m_tokens >= 1 (decode-sized
 *          counts run in one pass; larger ones in blocks of 8 tokens, each
 *          reading the weights again)
 *  qp      sweep-order codes from gptq_repack_sweep_order, 16-byte aligned
 *  scales, zeros  rows x G fp32 from gptq_quantize_layer (groups in sweep order)
 *  group_size 0 (per row), 32, 64 or 128; perm: sweep order (NULL = natural)
 *  Y       m_tokens x rows fp32
 *  half_sums  nonzero: for 4-bit codes, fp16 X and m_tokens <= 2, each 8-code word
 *          is summed in half precision (half2 FMA; relative rounding 2^-11 per
 *          step) before the fp32 grid step -- about half the instructions per code;
 *          otherwise (or 0) every sum is fp32.
 *  Errors: INVALID_ARG, UNSUPPORTED (other group sizes).
 */
gptq_status gptq_dequant_matmul(const void* X, int xdtype, int64_t m_tokens, int64_t cols,
                                int64_t ldx, const uint32_t* qp, const float* scales,
                                const float* zeros, int bits, int group_size,
                                const int32_t* perm, float* Y, int64_t rows, int half_sums,
                                void* stream);

/* Self-test of the failure detection (the pages have no counterpart).  Launches a
 * kernel whose bounded device wait is made to run out, so that a caller or a test
 * can check that the wait gives up, OR-s GPTQ_ERR_TIMEOUT into *dev_status and
 * returns with the context still usable:
 *   which = GPTQ_SELFTEST_MBARRIER: one CTA waits on a shared-memory mbarrier that
 *           nothing arrives on (the wait used by the tensor-core pipelines, with a
 *           shortened limit: well under a second);
 *   which = GPTQ_SELFTEST_GRID_BARRIER: two CTAs, of which one leaves without
 *           arriving at the software grid barrier of the persistent factorization;
 *           the other gives up after that barrier's own limit (about a second).
 * dev_status must be a device int32.  Returns GPTQ_ERR_INVALID_ARG for another
 * `which` or a NULL dev_status, GPTQ_ERR_CUDA if the launch fails. */
#define GPTQ_SELFTEST_MBARRIER 0
#define GPTQ_SELFTEST_GRID_BARRIER 1
gptq_status gptq_selftest_timeout(int which, int32_t* dev_status, void* stream);

/* Diagnostic (the pages have no counterpart): the number of polls after which a
 * wait in the tensor-core pipelines (the Hessian and the 3xTF32 products) gives up,
 * for kernels launched after this call; 0 restores the default (about a second).
 * With a small value the waits run out during normal work, so that a test can
 * check that such a kernel stops its producer and MMA issuer, waits for the copies
 * and MMAs it has in flight (those waits keep the default limit), frees its TMEM,
 * OR-s GPTQ_ERR_TIMEOUT into the status word and leaves the context usable.
 * Process-wide; returns the previous limit. */
uint32_t gptq_debug_set_wait_limit(uint32_t polls);

/* Human-readable name of a status code (static string). */
const char* gptq_status_string(int status);

/* Number of kernels this library has launched in the process (diagnostics). */
uint64_t gptq_launch_count(void);

/* Description of the most recent CUDA failure seen by the calling thread inside the
 * library (the call that returned GPTQ_ERR_CUDA), or "" if none.  Static per-thread
 * string, overwritten by the next failure. */
const char* gptq_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* GPTQ_H_ */
