/*
 * fa.h - C ABI of the exact tiled attention library (libfa.so), sm_100a.
 *
 * The library computes exact softmax attention
 *
 *     O = softmax(scale * Q K^T [+ causal mask | block mask]) V
 *
 * tile by tile with an online softmax, so the N x N score matrix never reaches
 * device memory, and the gradients of a scalar loss with respect to Q, K and V
 * by recomputing the attention tiles from the saved per-row log-sum-exp.
 *
 * Sources of the operations (pages on the method):
 *  - "FlashAttention-2: Faster Attention with Better Parallelism and Work
 *    Partitioning" (paper review), Abstract and "Proposed method": exact result,
 *    online-softmax tiling, parallelism over sequence length as well as batch and
 *    heads, causal masking by skipping blocks.
 *  - "Researchers at Stanford University Propose FlashAttention: Fast and
 *    Memory-Efficient Exact Attention with IO-Awareness" (summary), method
 *    paragraphs: inputs split into blocks with the softmax reduced progressively;
 *    the forward's softmax normalisation factor saved so that the backward
 *    recomputes attention on chip; block-sparse attention as a variant.
 *
 * Common conventions for every call
 *  - Tensors q, k, v, o, dO, dq, dk, dv: bfloat16, shape [B, H, N, d], contiguous,
 *    d innermost; element (b, h, n, c) at offset ((b*H + h)*N + n)*d + c.
 *  - lse: float32 [B, H, N]; lse[b,h,i] = ln sum_j exp(scale * q_i . k_j) over the
 *    keys visible to row i (natural log, scale and mask included); -INFINITY for
 *    a row that sees no key (a block mask whose tile row keeps nothing, or the
 *    causal mask with N_q > N_k, where the first N_q - N_k queries see no key).
 *  - All pointers are DEVICE pointers on the current device, except where noted.
 *    Every base pointer must be 16-byte aligned.
 *  - Supported sizes: B, H, N >= 1 (any N; the kernels work on 128-row tiles and
 *    the last tile of a sequence may be partial); d in {64, 96, 128} (d = 96 runs
 *    on the d = 128 kernels: the tensor-memory loads read zeros for columns 96..127,
 *    which leaves every product over the first 96 columns unchanged, and only 96
 *    columns are stored). B*H*Npad must fit in int32, where Npad = 128 * ceil(N / 128).
 *  - Causal: key j is visible to query i iff j <= i (top-left aligned; N_q = N_k).
 *  - Block mask (tile_mask): uint8 [nT, nT] device array with nT = ceil(N / 128),
 *    row-major, 1 = tile kept, 0 = tile skipped, shared by every (b, h); tile t
 *    covers rows 128 t .. min(128 t + 128, N) - 1. Within a kept tile every
 *    element is visible (the mask is not combined with causal).
 *  - Ownership: the caller owns every buffer. The library allocates and frees no
 *    device memory on these paths; scratch is caller-provided ("workspace").
 *  - Buffer sizes: each buffer must hold the elements its documented shape implies
 *    (q: B*H*N*d bf16, lse: B*H*N fp32, ...). The library receives only pointers and
 *    cannot check this (it checks the workspace's byte count, which is passed): a
 *    smaller buffer, or one on another device, is read or written out of bounds.
 *    The Python binding checks every tensor's shape, dtype, contiguity and device
 *    before it calls.
 *  - Asynchrony: each call only enqueues work on `stream` (a cudaStream_t, or
 *    NULL for the legacy default stream) and returns; no implicit synchronisation.
 *    Inputs must stay unmodified, and outputs unread, until the stream reaches
 *    that point.
 *  - Errors: arguments are checked synchronously before anything is enqueued; on
 *    a non-FA_OK return nothing has been written. A launch failure reported by the
 *    CUDA runtime returns FA_ERR_CUDA. Kernels never trap: a device-side wait that
 *    exceeds its time limit makes the kernel record FA_ERR_DEVICE_TIMEOUT in a
 *    library status word and return early; read it with fa_device_status().
 *  - Thread safety: calls may be made from several host threads on different
 *    streams.
 */
#ifndef FA_H_
#define FA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum fa_status {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = 1,     /* null pointer, non-positive size, non-finite scale */
  FA_ERR_UNSUPPORTED = 2,     /* d not in {64,96,128}, sizes beyond int32 rows, mask_block != 128 */
  FA_ERR_ALIGNMENT = 3,       /* a base pointer is not 16-byte aligned */
  FA_ERR_WORKSPACE = 4,       /* workspace too small */
  FA_ERR_CUDA = 5,            /* the CUDA runtime or driver reported an error */
  FA_ERR_DEVICE_TIMEOUT = 6   /* a kernel gave up waiting (see fa_device_status) */
} fa_status;

/* Memory layouts of q, k, v, o, dO, dq, dk, dv for fa_fwd_ex / fa_bwd_ex (lse is
 * [B, H, N] in both). Every other call uses FA_LAYOUT_BHND. */
enum {
  FA_LAYOUT_BHND = 0,  /* [B, H, N, d]: element (b, h, n, c) at ((b*H + h)*N + n)*d + c */
  FA_LAYOUT_BNHD = 1   /* [B, N, H, d]: element (b, n, h, c) at ((b*N + n)*H + h)*d + c */
};

/* Human-readable name of a status code (static string, never NULL). */
const char* fa_status_string(fa_status s);

/*
 * Forward (the review's "Proposed method": online-softmax tiling, sequence-length
 * parallelism; the summary's saved normalisation factor).
 *   q, k, v : [B,H,N,d] bf16 inputs.
 *   o       : [B,H,N,d] bf16 output, O = P V rounded to nearest-even.
 *   lse     : [B,H,N] fp32 output (see conventions).
 *   causal  : 0 = full attention, 1 = causal mask.
 *   scale   : softmax scale (usually 1/sqrt(d)); any finite value.
 */
fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                 int B, int H, int N, int d, int causal, float scale, void* stream);

/*
 * Forward with different query and key lengths (cross-attention, or a block of new
 * queries against a longer key sequence as in decoding). No counterpart on the
 * pages beyond the square problem; fa_fwd(..., N, ...) is fa_fwd_qk(..., N, N, ...).
 *   q, o    : [B,H,Nq,d] bf16;  k, v : [B,H,Nk,d] bf16;  lse : [B,H,Nq] fp32.
 *   causal  : 1 = key j is visible to query i iff j <= i + (Nk - Nq) (bottom-right
 *             alignment: the last query sees every key). With Nq > Nk the first
 *             Nq - Nk queries see no key: their O rows are 0 and lse -INFINITY.
 * Other arguments and rules as for fa_fwd.
 */
fa_status fa_fwd_qk(const void* q, const void* k, const void* v, void* o, float* lse,
                    int B, int H, int Nq, int Nk, int d, int causal, float scale, void* stream);

/*
 * fa_fwd_qk with a choice of memory layout: layout = FA_LAYOUT_BHND (as fa_fwd_qk)
 * or FA_LAYOUT_BNHD ([B, N, H, d] tensors, the row of (b, h, n) H*d elements after
 * that of (b, h, n - 1)). Any other value: FA_ERR_INVALID_ARG.
 */
fa_status fa_fwd_ex(const void* q, const void* k, const void* v, void* o, float* lse,
                    int B, int H, int Nq, int Nk, int d, int layout, int causal, float scale,
                    void* stream);

/*
 * Block-sparse forward (the summary's block-sparse paragraph): as fa_fwd without
 * the causal flag, restricted to the kept tiles of `tile_mask`. Skipped tiles
 * cost neither loads nor matrix products. mask_block must be 128.
 */
fa_status fa_fwd_blocksparse(const void* q, const void* k, const void* v, void* o, float* lse,
                             const uint8_t* tile_mask, int mask_block,
                             int B, int H, int N, int d, float scale, void* stream);

/*
 * Forward with dropout on the attention probabilities (dropout is named among the
 * element-wise O(N^2) operations of standard attention on the PagedAttention page,
 * section on bandwidth constraints; what follows is this library's definition).
 *   P = softmax(scale q k^T [causal]) as in fa_fwd; O = (P * M * 256 / t) V, where
 *   M is a 0/1 keep mask and t = round(256 (1 - p_drop)) in 1..256 (computed in
 *   double from p_drop): the drop probability is p_drop rounded to a multiple of
 *   1/256 and the kept entries are scaled so that E[O] is exact. lse is that of the
 *   softmax before dropout.
 *   M: element (b, h, i, j) is kept iff byte (j % 4) (least significant first) of
 *   word (i % 4) of Philox4x32-10 (Salmon et al., "Parallel Random Numbers: As Easy
 *   as 1, 2, 3", SC 2011) with counter (j / 4, i / 4, b H + h, offset) and key
 *   (seed mod 2^32, seed / 2^32) is below t. The same (seed, offset) passed to
 *   fa_bwd_dropout gives the gradients of the same function.
 *   p_drop : 0 <= p_drop < 1 with t >= 1, else FA_ERR_INVALID_ARG.
 *   d      : 64 or 128 (96: FA_ERR_UNSUPPORTED). Other arguments as for fa_fwd.
 */
fa_status fa_fwd_dropout(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N,
                         int d, int causal, float scale, float p_drop, uint64_t seed, uint32_t offset,
                         void* stream);

/*
 * Bytes of device scratch that fa_bwd / fa_bwd_blocksparse need for these sizes:
 * two fp32 [B,H,Npad] row arrays (D_i = sum_c dO_ic O_ic, and lse_i * log2 e;
 * Npad = 128 * ceil(N / 128), so each tile's rows are one run), each rounded up to
 * 256 bytes: 2 * round_up_256(4 * B*H*Npad). Returns 0 for non-positive sizes.
 */
size_t fa_bwd_workspace_bytes(int B, int H, int N, int d);

/*
 * Backward (the summary's method paragraph: attention recomputed on chip from
 * the saved normalisation factor). Gradients of L = sum(O * dO):
 *   dv = P^T dO, dS = P * (dO V^T - D), dq = scale dS K, dk = scale dS^T Q.
 *   q, k, v, o, lse : the forward's inputs and outputs (o and lse from fa_fwd
 *                     with the same causal flag and scale).
 *   dO              : [B,H,N,d] bf16 upstream gradient.
 *   dq, dk, dv      : [B,H,N,d] bf16 outputs.
 *   workspace       : device scratch of at least fa_bwd_workspace_bytes(B,H,N,d)
 *                     bytes, 256-byte aligned; its contents on entry do not
 *                     matter; it must not be shared with a concurrent call.
 * All three gradients are deterministic (no atomics): dk and dv come from one pass
 * over the query tiles per key tile, dq from one pass over the key tiles per query
 * tile (which recomputes the scores and dP it needs).
 */
fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
                 const void* dO, void* dq, void* dk, void* dv,
                 void* workspace, size_t workspace_bytes,
                 int B, int H, int N, int d, int causal, float scale, void* stream);

/*
 * Backward of fa_fwd_qk: dq [B,H,Nq,d], dk and dv [B,H,Nk,d]; o, lse and dO have Nq
 * rows. The workspace holds per-query rows: fa_bwd_workspace_bytes(B, H, Nq, d).
 * fa_bwd(..., N, ...) is fa_bwd_qk(..., N, N, ...).
 */
fa_status fa_bwd_qk(const void* q, const void* k, const void* v, const void* o, const float* lse,
                    const void* dO, void* dq, void* dk, void* dv,
                    void* workspace, size_t workspace_bytes,
                    int B, int H, int Nq, int Nk, int d, int causal, float scale, void* stream);

/* fa_bwd_qk with a choice of memory layout (as fa_fwd_ex; lse stays [B, H, Nq]). */
fa_status fa_bwd_ex(const void* q, const void* k, const void* v, const void* o, const float* lse,
                    const void* dO, void* dq, void* dk, void* dv,
                    void* workspace, size_t workspace_bytes,
                    int B, int H, int Nq, int Nk, int d, int layout, int causal, float scale,
                    void* stream);

/* Block-sparse backward: fa_bwd restricted to the kept tiles of `tile_mask`. */
fa_status fa_bwd_blocksparse(const void* q, const void* k, const void* v, const void* o,
                             const float* lse, const void* dO, void* dq, void* dk, void* dv,
                             void* workspace, size_t workspace_bytes,
                             const uint8_t* tile_mask, int mask_block,
                             int B, int H, int N, int d, float scale, void* stream);

/*
 * The three launches that make up fa_bwd / fa_bwd_blocksparse, for callers that
 * schedule or time them separately. On one stream,
 *   fa_bwd_preprocess; fa_bwd_dkdv; fa_bwd_dq
 * is exactly fa_bwd (tile_mask = NULL) or fa_bwd_blocksparse (tile_mask set).
 * Arguments have the meanings given for fa_bwd; the workspace must be the same
 * buffer for all three. fa_bwd_dkdv and fa_bwd_dq only read the workspace and may
 * run in either order (or concurrently) after fa_bwd_preprocess.
 *   fa_bwd_preprocess : D_i = sum_c dO_ic O_ic and lse_i log2(e) into the workspace.
 *   fa_bwd_dkdv       : dk and dv. tile_mask may be NULL (then `causal` applies)
 *                       or a block mask (then causal must be 0, mask_block 128).
 *   fa_bwd_dq         : dq (same mask rules).
 */
fa_status fa_bwd_preprocess(const void* o, const void* dO, const float* lse, void* workspace,
                            size_t workspace_bytes, int B, int H, int N, int d, void* stream);
fa_status fa_bwd_dkdv(const void* q, const void* k, const void* v, const void* dO, void* dk, void* dv,
                      const void* workspace, size_t workspace_bytes,
                      const uint8_t* tile_mask, int mask_block,
                      int B, int H, int N, int d, int causal, float scale, void* stream);
fa_status fa_bwd_dq(const void* q, const void* k, const void* v, const void* dO, void* dq,
                    const void* workspace, size_t workspace_bytes,
                    const uint8_t* tile_mask, int mask_block,
                    int B, int H, int N, int d, int causal, float scale, void* stream);

/*
 * Fused backward: the same gradients as fa_bwd from ONE kernel per call instead of two,
 * executing five matrix products per (key tile, query tile) pair instead of seven (the
 * summary's recomputation: S and dP are formed once per pair; the deterministic path
 * forms them a second time for dq). dQ_i's share from each key tile is added in fp32
 * into an accumulator in the workspace with the tensor memory accelerator's bulk
 * reduce-add, then converted: dq = bf16(scale * accumulator).
 *   NOT bit-reproducible: the key tiles add into a dq row in an order that varies from
 *   run to run (fp32 sums; dk and dv are deterministic). Use fa_bwd when run-to-run
 *   identical gradients are required.
 *   workspace : at least fa_bwd_fused_workspace_bytes(B,H,N,d) bytes, 256-byte
 *               aligned (the two row arrays of fa_bwd, then the fp32 accumulator
 *               [B*H, Npad, 64 (d = 64) or 128 (d = 96, 128)]); contents on entry do
 *               not matter; not to be shared with a concurrent call.
 * Other arguments, results and rules as for fa_bwd. No dropout variant.
 */
size_t fa_bwd_fused_workspace_bytes(int B, int H, int N, int d);
fa_status fa_bwd_fused(const void* q, const void* k, const void* v, const void* o, const float* lse,
                       const void* dO, void* dq, void* dk, void* dv,
                       void* workspace, size_t workspace_bytes,
                       int B, int H, int N, int d, int causal, float scale, void* stream);

/*
 * fa_bwd_fused with query and key lengths of their own (as fa_bwd_qk), a memory layout
 * (as fa_bwd_ex) and an optional block mask (tile_mask NULL, or as fa_bwd_blocksparse
 * with causal = 0, Nq = Nk and mask_block = 128; else FA_ERR_UNSUPPORTED). The
 * workspace holds per-query rows: fa_bwd_fused_workspace_bytes(B, H, Nq, d).
 */
fa_status fa_bwd_fused_ex(const void* q, const void* k, const void* v, const void* o, const float* lse,
                          const void* dO, void* dq, void* dk, void* dv,
                          void* workspace, size_t workspace_bytes,
                          const uint8_t* tile_mask, int mask_block,
                          int B, int H, int Nq, int Nk, int d, int layout, int causal, float scale,
                          void* stream);

/*
 * The three launches that make up fa_bwd_fused (tile_mask NULL) or its block-sparse
 * form, for callers that schedule or time them separately; same workspace for all
 * three, in this order on one stream:
 *   fa_bwd_fused_preprocess : the row arrays of fa_bwd_preprocess, and the fp32 dQ
 *                             accumulator set to zero.
 *   fa_bwd_fused_main       : dk and dv written; dq's shares added into the
 *                             accumulator (mask rules as fa_bwd_dkdv).
 *   fa_bwd_fused_dq         : dq [B,H,N,d] bf16 = bf16(scale * accumulator).
 */
fa_status fa_bwd_fused_preprocess(const void* o, const void* dO, const float* lse, void* workspace,
                                  size_t workspace_bytes, int B, int H, int N, int d, void* stream);
fa_status fa_bwd_fused_main(const void* q, const void* k, const void* v, const void* dO, void* dk, void* dv,
                            void* workspace, size_t workspace_bytes,
                            const uint8_t* tile_mask, int mask_block,
                            int B, int H, int N, int d, int causal, float scale, void* stream);
fa_status fa_bwd_fused_dq(void* dq, const void* workspace, size_t workspace_bytes,
                          int B, int H, int N, int d, float scale, void* stream);

/*
 * Backward without caller-provided scratch (no counterpart on the pages: this is
 * an interface convenience, not part of the method).
 *
 * For callers that cannot allocate device memory when they call the backward: a
 * plugin whose host application owns all device memory and hands it only the
 * input and output buffers, or a latency-critical loop that must not pay the
 * implicit device synchronisation of cudaMalloc/cudaFree. Same arguments and
 * results as fa_bwd / fa_bwd_blocksparse (tile_mask NULL or a 128-granular block
 * mask with causal = 0), but the fp32 scratch (two per-row arrays) lives in one
 * array compiled into the library: FA_BWD_NOALLOC_SCRATCH_BYTES bytes of device
 * memory on every GPU that loads the library, held until the process exits.
 *  - Sizes: needs fa_bwd_workspace_bytes(B,H,N,d) <= FA_BWD_NOALLOC_SCRATCH_BYTES,
 *    i.e. B*H*Npad <= 1,048,576 rows (any d); larger sizes return FA_ERR_WORKSPACE
 *    and enqueue nothing.
 *  - Allocation: none. No cudaMalloc, cudaFree or allocating library call.
 *  - Set-up: the first call on a device (with that device current) looks up the
 *    array's device address once; make that first call before any stream
 *    capture on that device.
 *  - Sharing: every call on a device uses the same array and leaves its contents
 *    behind; each call re-initialises what it reads. Calls whose work overlaps on
 *    the GPU (different streams, or several threads) race on the array: serialise
 *    them (e.g. one stream).
 */
#define FA_BWD_NOALLOC_SCRATCH_BYTES (8u * 1024u * 1024u)
fa_status fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const float* lse,
                         const void* dO, void* dq, void* dk, void* dv,
                         const uint8_t* tile_mask, int mask_block,
                         int B, int H, int N, int d, int causal, float scale, void* stream);

/*
 * Backward of fa_fwd_dropout (same p_drop, seed and offset, and its o and lse):
 * dV = P~^T dO, dP = (dO V^T) * M * 256 / t, dS = P * (dP - D), dQ = scale dS K,
 * dK = scale dS^T Q with P~ = P * M * 256 / t and D = rowsum(dO * O). Arguments,
 * workspace and rules as for fa_bwd, plus those of fa_fwd_dropout.
 */
fa_status fa_bwd_dropout(const void* q, const void* k, const void* v, const void* o, const float* lse,
                         const void* dO, void* dq, void* dk, void* dv, void* workspace, size_t workspace_bytes, int B,
                         int H, int N, int d, int causal, float scale, float p_drop, uint64_t seed, uint32_t offset,
                         void* stream);

/*
 * Attention over a key sequence split into blocks (the sequence-parallel ring, where
 * each GPU holds one block of queries, keys and values and the key/value blocks
 * travel around the GPUs). Softmax attention over the union of two key sets is the
 * log-sum-exp-weighted mean of the two partial results: the combination the review's
 * "Proposed method" performs tile by tile with its online softmax, and that the
 * summary's saved normalisation factor makes possible afterwards; these calls do it
 * block by block. Splitting one sequence across GPUs is not on the pages (they split
 * it across the thread blocks of one GPU); fa_accumulate_bf16 and fa_to_bf16 are its
 * plumbing and have no counterpart there.
 *
 * fa_merge_partial: merges a partial result (o_part bf16 [rows, d], lse_part fp32
 * [rows], as written by fa_fwd for one key block) into the running one (o_acc fp32
 * [rows, d], lse_acc fp32 [rows], updated in place):
 *   lse' = ln(e^lse_acc + e^lse_part),
 *   o'   = o_acc e^(lse_acc - lse') + o_part e^(lse_part - lse').
 * Start from o_acc = 0 and lse_acc = -INFINITY; a row with both -INFINITY stays
 * o = 0, lse = -INFINITY. rows = B*H*N_q; d 64 or 128 (else FA_ERR_UNSUPPORTED);
 * o_acc and o_part 16-byte aligned (FA_ERR_ALIGNMENT). Device pointers; async.
 */
fa_status fa_merge_partial(float* o_acc, float* lse_acc, const void* o_part, const float* lse_part, long long rows,
                           int d, void* stream);

/*
 * fa_fwd_merge: the attention of q against one key block (k, v), merged straight into the
 * running result (o_acc fp32 [B,H,N,d], lse_acc fp32 [B,H,N], updated in place) by the
 * kernel's epilogue with the rule of fa_merge_partial, without rounding the block's
 * partial O to bf16 first. Query and key blocks have N rows each; causal = 1 applies the
 * causal mask within the pair (the diagonal block of a longer sequence), else every key
 * is visible. d 64 or 128 (else FA_ERR_UNSUPPORTED); a row that sees no key of the block
 * is left unchanged. Other arguments and rules as for fa_fwd.
 */
fa_status fa_fwd_merge(const void* q, const void* k, const void* v, float* o_acc, float* lse_acc, int B, int H,
                       int N, int d, int causal, float scale, void* stream);

/*
 * fa_bwd_fused_main with fp32 outputs: dk and dv are fp32 [B,H,N,d] (a key block's share
 * of the gradients of a longer sequence, to be accumulated in fp32 without a bf16
 * rounding). The workspace's dQ accumulator receives dq's share as in fa_bwd_fused_main,
 * so successive calls on one workspace (after one fa_bwd_fused_preprocess) add up the
 * shares of several key blocks. d 64, 96 or 128 (256: FA_ERR_UNSUPPORTED); no mask.
 */
fa_status fa_bwd_fused_main_f32(const void* q, const void* k, const void* v, const void* dO, float* dk, float* dv,
                                void* workspace, size_t workspace_bytes, int B, int H, int N, int d, int causal,
                                float scale, void* stream);

/* acc[i] += x[i] for i < n (fp32; device pointers, 16-byte aligned; n a multiple of 8). */
fa_status fa_accumulate_f32(float* acc, const float* x, long long n, void* stream);

/*
 * acc[i] = (overwrite ? 0 : acc[i]) + x[i] for i < n: fp32 accumulation of a bf16
 * partial gradient (device pointers, both 16-byte aligned; n a multiple of 8).
 */
fa_status fa_accumulate_bf16(float* acc, const void* x, long long n, int overwrite, void* stream);

/* out[i] = bf16(in[i]), round to nearest even (n a multiple of 8; 16-byte aligned). */
fa_status fa_to_bf16(void* out, const float* in, long long n, void* stream);

/*
 * Synchronises `stream`, then returns and clears the library's device status
 * word for the current device: FA_OK, or FA_ERR_DEVICE_TIMEOUT if a kernel since
 * the last call gave up on a wait. *detail (if non-NULL, host pointer) receives
 * a kernel-specific code naming the wait that expired (0 if none).
 */
fa_status fa_device_status(void* stream, int* detail);

/*
 * Diagnostic: y[i] = 2^x[i] for i < n, evaluated on the device by one of the two
 * exponential paths the kernels split every score tile between. mode 0: the
 * special-function unit (ex2.approx); mode 1: the library's own polynomial
 * (round-to-nearest range reduction, cubic fitted on [-1/2, 1/2], max relative
 * error about 1e-4; inputs below -126 give about 1e-38). x and y are device
 * arrays of n floats, n >= 0; asynchronous on `stream` like every call here.
 */
fa_status fa_debug_exp2(const float* x, float* y, int n, int mode, void* stream);

/*
 * Diagnostic for the bounded waits behind FA_ERR_DEVICE_TIMEOUT: launches one block
 * of two warps on `stream`. Warp 0 waits, with a limit of timeout_us microseconds,
 * on a shared-memory barrier that nothing completes; when the limit passes it
 * records FA_ERR_DEVICE_TIMEOUT with detail 901 in the status word and raises the
 * block's abort flag. Warp 1 waits on a second such barrier with a limit 64 times
 * longer and leaves when it sees the flag, as the kernels' other roles do. Nothing
 * traps and the context stays usable; read the result with fa_device_status().
 *   timeout_us : 1 .. 100000, else FA_ERR_INVALID_ARG (nothing launched).
 *   out        : device array of 3 ints, or NULL (4-byte aligned, else
 *                FA_ERR_ALIGNMENT). out[0] = 1 if warp 0 gave up at its limit;
 *                out[1] = 1 if warp 1 left on the flag before its own limit;
 *                out[2] = how long warp 0 waited, in microseconds.
 */
fa_status fa_debug_wait_timeout(int timeout_us, int* out, void* stream);

/*
 * Test hook for the bounded waits of the attention kernels themselves. mode 1: every
 * forward, dK/dV and dQ launch made after this call, by any host thread on any
 * stream, runs with a TMA producer that issues no copies and with a wait limit of
 * timeout_us microseconds (1 .. 100000) instead of the usual 4 s. Its other roles
 * wait for tiles that never arrive, give up at the limit, record
 * FA_ERR_DEVICE_TIMEOUT and the site of the wait (forward 101..110, backward
 * 201..211) in the status word, and the kernel returns through its normal teardown
 * with its outputs unwritten. No copy or matrix product is in flight at any time.
 * The backward pre-pass has no waits and runs normally. mode 0: normal launches
 * again (timeout_us ignored). Any other mode or limit: FA_ERR_INVALID_ARG, the
 * setting unchanged. Never call this while other threads launch work they need.
 */
fa_status fa_debug_stall_producer(int mode, int timeout_us);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
int fa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FA_H_ */
