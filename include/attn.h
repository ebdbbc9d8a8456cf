/*
 * attn.h -- C ABI of the B200 (sm_100a) causal softmax attention library.
 *
 * The library computes batched, multi-head softmax attention (causal or full)
 * and its backward pass, dQ, dK, dV from Q, K, V, O, dO and the per-row
 * log-sum-exp. The scores are recomputed tile by tile inside the backward from
 * Q, K and one saved number per row, LSE = m + log z, so no N x N tensor is
 * ever written to device memory (ddx issue #243, "Attention's gradient: a
 * softmax shift's backward computed twice, and recomputing scores instead of
 * saving them", item 2). The max-shift's gradient is dropped, since it
 * cancels in w / z (same issue, item 1); the backward uses the row term
 * D_i = sum_c dO_ic O_ic instead.
 *
 * Beyond that: block-sparse masks (attn_*_masked), arbitrary row strides
 * (attn_*_strided), N_q != N_k with a query position offset (attn_*_rect)
 * and the backward-over-backward (attn_bwd_bwd), each declared below with its
 * own conventions.
 *
 * Layout. Unless an entry point says otherwise, every matrix argument is a
 * DEVICE pointer to a contiguous [B][H][N][d] row-major array (batch, head,
 * position, channel), of the
 * element type `dtype` (ATTN_F32: float, ATTN_BF16: bfloat16 bits). LSE is a
 * device [B][H][N] float array in natural-log units: LSE_i = m_i + ln z_i of
 * the SCALED scores s_ij = scale * q_i . k_j (the scale is applied before the
 * max, as in ddx issue #217's repro, `SUM(q.val * k.val) / 2.0`). With
 * causal != 0 position i sees keys j <= i (diagonal included, the repro's
 * `WHERE q.pos >= k.pos`); causal == 0 is full attention. N_q == N_k == N
 * except in attn_*_rect.
 *
 * Ownership. The caller allocates and frees every buffer, the backward's
 * workspace included. The library never allocates or frees device memory,
 * never synchronises the host with the device (except attn_last_status),
 * and enqueues all work on `stream` (a cudaStream_t passed as void*; NULL is
 * the legacy default stream).
 *
 * Errors. Arguments are checked before anything is launched:
 *   null pointers, B, H, N <= 0, d <= 0, non-finite scale, tensor pointers
 *   not 16-byte aligned (bf16) or 4-byte aligned (f32), an LSE array or a
 *   workspace not 16-byte aligned, a workspace smaller than
 *   attn_bwd_workspace_bytes -> ATTN_ERR_INVALID
 *   (dtype, d) outside the built set: bf16 with d in {32, 64, 128}, f32 with
 *   1 <= d <= 128 -> ATTN_ERR_UNSUPPORTED
 *   a failed launch or a non-sm_100 device -> ATTN_ERR_CUDA
 * Device-side waits are bounded; a wait that runs out writes ATTN_ERR_TIMEOUT
 * into a status word (the workspace's for the backward, a library-owned one
 * for the forward) and the kernel returns without trapping. Input VALUES are
 * not validated: NaN and infinities propagate as IEEE arithmetic carries them.
 *
 * Debug build. The same sources compiled with ATTN_DEBUG (build.py --debug:
 * libcsa_attn_debug.so, same symbols) check tile coordinates and row indices
 * in the kernels before the global accesses a thread makes -- a failed check
 * writes ATTN_ERR_BOUNDS into the status word and skips the access, never a
 * trap -- and fill the outputs of attn_fwd / attn_bwd / attn_fwd_rect /
 * attn_bwd_rect / attn_bwd_bwd with NaN (on the call's stream) before their
 * kernels run, so that an element no kernel writes shows up.
 */
#ifndef CSA_ATTN_H_
#define CSA_ATTN_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  ATTN_OK = 0,
  ATTN_ERR_INVALID = -1,
  ATTN_ERR_UNSUPPORTED = -2,
  ATTN_ERR_CUDA = -3,
  ATTN_ERR_TIMEOUT = -4,
  ATTN_ERR_BOUNDS = -5 /* debug builds only: a device-side bounds check failed */
} attn_status;

typedef enum { ATTN_F32 = 0, ATTN_BF16 = 1 } attn_dtype;

/*
 * Forward: O = softmax(scale * Q K^T, causal filter) V and LSE = m + ln z per
 * row (ddx issue #217's repro: the `scores`, `weights`, `norm` and `heads`
 * steps; LSE is the saved number of ddx issue #243, item 2).
 *   q, k, v : in,  [B][H][N][d] of dtype
 *   o       : out, [B][H][N][d] of dtype
 *   lse     : out, [B][H][N] float
 * Returns an attn_status.
 */
int attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
             int N, int d, int causal, float scale, int dtype, void* stream);

/*
 * Bytes of device workspace attn_bwd needs for this shape: a status word, the
 * row terms D and LSE (padded to whole 128-row tiles) and, for bf16, an fp32
 * dQ accumulator. Returns 0 for arguments attn_bwd would reject.
 */
size_t attn_bwd_workspace_bytes(int B, int H, int N, int d, int dtype);

/*
 * Backward: given dO = dL/dO, writes
 *   dV = P^T dO,  dP = dO V^T,  D_i = sum_c dO_ic O_ic,
 *   dS = P o (dP - D),  dQ = scale dS K,  dK = scale dS^T Q
 * (ddx PR #162, "perf(ddx-ad): transpose causal attention's contractions
 * without their joins", "What changed": transpose p = w / z per score, then
 * p @ v; ddx issue #243 items 1-2 for dropping the shift and using D).
 *   q, k, v, o, dout : in,  [B][H][N][d] of dtype (o from attn_fwd)
 *   lse              : in,  [B][H][N] float (from attn_fwd)
 *   dq, dk, dv       : out, [B][H][N][d] of dtype
 *   workspace        : device scratch of >= attn_bwd_workspace_bytes bytes,
 *                      16-byte aligned; contents need not be initialised
 * Runs three stream-ordered kernels: attn_bwd_preprocess, attn_bwd_main and
 * (bf16 only) attn_bwd_dq_convert.
 */
int attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
             const float* lse, void* dq, void* dk, void* dv, int B, int H, int N, int d,
             int causal, float scale, int dtype, void* workspace, size_t workspace_bytes,
             void* stream);

/*
 * Block-sparse attention: the causal / full filter replaced by a block mask
 * over 128 x 128 tiles of (query, key) positions -- the generalisation of the
 * mask that ddx PR #162 ("perf(ddx-ad): transpose causal attention's
 * contractions without their joins", "What changed") applies as a filter on
 * the grouping keys, and of its tile skipping. bf16 only.
 *   block_mask : in, DEVICE [T][T] bytes, T = ceil(N / 128), row-major by
 *                query tile: block_mask[a * T + b] describes query rows
 *                [128a, 128a+128) against key columns [128b, 128b+128):
 *                  0  no score of the tile takes part (the tile is skipped),
 *                  1  every score takes part,
 *                  2  a score takes part when its key's index inside the tile
 *                     is at most its query's (the causal filter's diagonal
 *                     tile; causal attention is 1 below the diagonal, 2 on
 *                     it, 0 above). Other values act as 1.
 *                Shared by every (batch, head). Read, not written; owned by
 *                the caller and must stay valid until the kernels finish.
 * Rows whose query keeps no score (a query tile with only 0 entries) get
 * O = 0 and LSE = -inf (the log of an empty sum), and zero gradients; keys
 * that no query keeps get dK = dV = 0.
 * Other arguments, layouts, ownership and checks as attn_fwd / attn_bwd;
 * block_mask == NULL -> ATTN_ERR_INVALID, dtype f32 -> ATTN_ERR_UNSUPPORTED.
 */
int attn_fwd_masked(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                    int H, int N, int d, const unsigned char* block_mask, float scale, int dtype,
                    void* stream);
int attn_bwd_masked(const void* q, const void* k, const void* v, const void* o,
                    const void* dout, const float* lse, void* dq, void* dk, void* dv, int B,
                    int H, int N, int d, const unsigned char* block_mask, float scale, int dtype,
                    void* workspace, size_t workspace_bytes, void* stream);

/*
 * Strided layouts: q, k, v, o, dout, dq, dk, dv given as [B][H][N][d] views
 * of arbitrary row strides (the channel stride is 1), so that the
 * (sequence, position, head, channel) tables of ddx issue #217 ("Backward of
 * batched attention builds a contraction over every pair of sequences and
 * heads", the repro's `q`, `k`, `v` tables and its JAX restatement), or a
 * packed [B][N][3][H][d] projection output, are consumed without a permute.
 *   qkv_strides : in, HOST array {s_b, s_h, s_n} of element strides for q, k,
 *                 v and for dq, dk, dv: row n of head (b, h) of q starts at
 *                 q + b*s_b + h*s_h + n*s_n.
 *   o_strides   : in, HOST array {s_b, s_h, s_n} for o and dout.
 * Each stride must be > 0 and < 2^36 and s_n >= d; for bf16 each must be a
 * multiple of 8 elements (16 bytes). Rows of the outputs must not overlap.
 * Contiguous [B][H][N][d] is {H*N*d, N*d, d}; [B][N][H][d] is
 * {N*H*d, d, H*d}. LSE stays a contiguous [B][H][N] fp32 array.
 * Everything else (arguments, results, workspace, checks, statuses) as
 * attn_fwd / attn_bwd; a NULL or out-of-range stride array -> ATTN_ERR_INVALID.
 */
int attn_fwd_strided(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                     int H, int N, int d, const long long* qkv_strides,
                     const long long* o_strides, int causal, float scale, int dtype,
                     void* stream);
int attn_bwd_strided(const void* q, const void* k, const void* v, const void* o,
                     const void* dout, const float* lse, void* dq, void* dk, void* dv, int B,
                     int H, int N, int d, const long long* qkv_strides,
                     const long long* o_strides, int causal, float scale, int dtype,
                     void* workspace, size_t workspace_bytes, void* stream);

/*
 * N_q != N_k: N_q query rows attending to N_k keys. Query row r stands for
 * position q_offset + r and key j for position j; with causal != 0 a score is
 * kept when the query's position is at least the key's -- the repro's
 * `WHERE q.pos >= k.pos` of ddx issue #217 ("Backward of batched attention
 * builds a contraction over every pair of sequences and heads") read on
 * absolute positions. q_offset = N_k - N_q is the usual key-value-cache
 * shape (the last N_q positions); q_offset is ignored without the filter.
 *   q, o, dout, dq : [B][H][N_q][d] of dtype, contiguous
 *   k, v, dk, dv   : [B][H][N_k][d] of dtype, contiguous
 *   lse            : [B][H][N_q] float
 *   workspace      : >= attn_bwd_workspace_bytes(B, H, N_q, d, dtype) bytes
 * n_q, n_k >= 1 and 0 <= q_offset <= 2^30, else ATTN_ERR_INVALID; every row
 * then keeps key 0, so no row is empty. Keys after the last query's position
 * get dK = dV = 0. Everything else (dtypes, head sizes, checks, statuses) as
 * attn_fwd / attn_bwd, which are the case n_q = n_k, q_offset = 0.
 */
int attn_fwd_rect(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                  int H, int n_q, int n_k, int d, int q_offset, int causal, float scale,
                  int dtype, void* stream);
int attn_bwd_rect(const void* q, const void* k, const void* v, const void* o, const void* dout,
                  const float* lse, void* dq, void* dk, void* dv, int B, int H, int n_q, int n_k,
                  int d, int q_offset, int causal, float scale, int dtype, void* workspace,
                  size_t workspace_bytes, void* stream);

/*
 * Backward-over-backward (the FlashBoB listing, "Approaching I/O-optimality
 * for Approximate Attention": exact differentiation through attention's
 * backward pass). With (dQ, dK, dV) the first backward of (q, k, v, dout)
 * and uq, uk, uv cotangents on them, computes the gradients of
 *     L2 = <uq, dQ> + <uk, dK> + <uv, dV>
 * with respect to q, k, v and dout:
 *   gq, gk, gv, gdout : out, DEVICE [B][H][N][d], same dtype as q.
 * o and lse are the forward's outputs for (q, k, v) (attn_fwd). The scores
 * are recomputed tile by tile in two passes (two row-wise scalars first,
 * then the gradients); nothing N x N is stored. dtype ATTN_F32 (CUDA-core
 * FFMA kernels, 1 <= d <= 128, pointers 4-byte aligned) or ATTN_BF16
 * (tensor-core kernels, bf16 in and out with fp32 accumulation, d in
 * {32, 64, 128}, pointers 16-byte aligned); contiguous [B][H][N][d]; lse
 * and workspace 16-byte aligned.
 *   workspace : DEVICE scratch of >= attn_bwd_bwd_workspace_bytes bytes
 *               (0 for an unsupported shape or dtype).
 * Three stream-ordered kernels: the backward's preprocess (D, padded LSE),
 * a query-row kernel (row scalars, gq, gdout), a key-row kernel (gk, gv).
 */
size_t attn_bwd_bwd_workspace_bytes(int B, int H, int N, int d, int dtype);
int attn_bwd_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
                 const float* lse, const void* uq, const void* uk, const void* uv, void* gq,
                 void* gk, void* gv, void* gdout, int B, int H, int N, int d, int causal,
                 float scale, int dtype, void* workspace, size_t workspace_bytes, void* stream);

/*
 * The three stages attn_bwd runs, exposed so a caller can time or overlap them
 * separately. Same arguments and checks as attn_bwd; they must be enqueued in
 * this order on one stream with the same workspace.
 *   preprocess : D_i = sum_c dO_ic O_ic, the padded LSE copy, zeroes the dQ
 *                accumulator and the status word
 *   main       : the tile loop (scores recomputed from Q, K, LSE; dV, dK; dQ
 *                partial sums). For f32 it also writes dq.
 *   dq_convert : dq = scale * accumulator, rounded to bf16 (bf16 only; a
 *                no-op returning ATTN_OK for f32)
 *   main_masked: the main stage of attn_bwd_masked (block_mask as there; bf16
 *                only), between the same preprocess and dq_convert
 */
int attn_bwd_preprocess(const void* o, const void* dout, const float* lse, int B, int H, int N,
                        int d, int dtype, void* workspace, size_t workspace_bytes, void* stream);
int attn_bwd_main(const void* q, const void* k, const void* v, const void* dout, void* dq,
                  void* dk, void* dv, int B, int H, int N, int d, int causal, float scale,
                  int dtype, void* workspace, size_t workspace_bytes, void* stream);
int attn_bwd_dq_convert(void* dq, int B, int H, int N, int d, float scale, int dtype,
                        void* workspace, size_t workspace_bytes, void* stream);
int attn_bwd_main_masked(const void* q, const void* k, const void* v, const void* dout, void* dq,
                         void* dk, void* dv, int B, int H, int N, int d,
                         const unsigned char* block_mask, float scale, int dtype, void* workspace,
                         size_t workspace_bytes, void* stream);

/*
 * Reads the backward's device status word from `workspace` (synchronises the
 * calling thread with the device). ATTN_OK, or ATTN_ERR_TIMEOUT if a bounded
 * device wait ran out during the last attn_bwd on this workspace.
 */
int attn_last_status(const void* workspace);

/*
 * Same for the forward: reads (and clears) the library's forward status word
 * on the current device. Synchronises.
 */
int attn_fwd_last_status(void);

/* Static, human-readable name of a status code. */
const char* attn_status_string(int status);

/*
 * Failure-detection hook for tests. Arms a one-shot fault for the NEXT bf16
 * attn_bwd_main (or attn_bwd) or bf16 attn_bwd_bwd call in this process: that
 * launch withholds the signal that its first score tile (backward-over-
 * backward: the rows kernel's first score quarter) is ready and bounds each
 * of its device waits by `wait_limit_cycles` SM clock cycles, so the waits
 * run out, the kernel writes ATTN_ERR_TIMEOUT into the workspace status word,
 * releases its tensor memory and returns. No fault, trap or unbounded wait is involved; the
 * outputs of that call are undefined. Returns ATTN_ERR_INVALID for
 * wait_limit_cycles == 0.
 */
int attn_test_arm_timeout(unsigned long long wait_limit_cycles);

/*
 * Test hook for the forward's exponentials (not part of the method; the pages
 * have no counterpart): for n DEVICE floats x, writes 2^x computed the two
 * ways the bf16 forward computes it -- on the FMA pipe by Cody-Waite range
 * reduction and a degree-3 polynomial (`poly`) and by the MUFU ex2.approx
 * instruction (`mufu`) -- so that tests can bound the polynomial against
 * the hardware instruction and exact values. Device pointers, enqueued on
 * `stream`; NULL pointers or n < 0 -> ATTN_ERR_INVALID.
 */
int attn_test_exp2(const float* x, float* poly, float* mufu, int n, void* stream);

/*
 * Backward without any allocation, for callers that cannot call cudaMalloc:
 * code running inside a host framework whose device memory is reserved by that
 * framework's own pool (a plugin or custom operator that may not allocate),
 * or latency-critical code that cannot afford an allocation, which may also
 * synchronise the device. The pages have no counterpart: this is a
 * deployment variant of attn_bwd, not part of the method.
 *
 * Same arguments, layout, results and checks as attn_bwd, minus the
 * workspace: the scratch comes from a fixed device array of
 * ATTN_BWD_NOALLOC_SCRATCH_BYTES compiled into the library, which every GPU
 * that loads the library holds until the process exits. Shapes whose
 * attn_bwd_workspace_bytes exceeds that size are rejected with
 * ATTN_ERR_INVALID before anything is launched (for bf16 the need is about
 * 4 * B * H * N * (d + 2) bytes).
 *
 * The first call on each device looks up the array's device address (with that
 * device current) and caches it; make that first call before any stream
 * capture. All calls share the one array and it keeps the last call's
 * contents (each call re-zeroes what must start at zero), so calls that
 * overlap on the same GPU race: serialise them. The address is cached per
 * device together with the CUDA context it was found in; a call from a new
 * context (after a device reset, say) looks it up again. Device-side
 * timeouts are recorded in the array's status word: read it with
 * attn_bwd_noalloc_last_status. Returns an attn_status.
 */
#define ATTN_BWD_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)
int attn_bwd_noalloc(const void* q, const void* k, const void* v, const void* o,
                     const void* dout, const float* lse, void* dq, void* dk, void* dv, int B,
                     int H, int N, int d, int causal, float scale, int dtype, void* stream);

/*
 * The status word of the last attn_bwd_noalloc on the current device (as
 * attn_last_status reads a workspace's): ATTN_OK, or ATTN_ERR_TIMEOUT if a
 * bounded device wait of that call ran out. Synchronises the calling thread
 * with the device; allocates nothing.
 */
int attn_bwd_noalloc_last_status(void);

#ifdef __cplusplus
}
#endif

#endif /* CSA_ATTN_H_ */
