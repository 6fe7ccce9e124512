/*
 * fa.h -- C ABI of libfa_b200.so: exact attention forward on NVIDIA B200
 * (sm_100a).
 *
 * The operation is the pages' "standard attention" (Flash Attention | Hermes
 * Skill, Workflow 1, Step 2): for every batch b, head h and query row i
 *
 *     S_ij   = scale * sum_d Q[b,i,h,d] * K[b,j,h,d]
 *     O[b,i,h,:] = sum_j softmax_j(S_ij over visible j) * V[b,j,h,:]
 *     LSE[b,h,i] = ln sum_{visible j} exp(S_ij)
 *
 * computed tile by tile with an online softmax so the N_q x N_k scores never
 * reach device memory (FlashAttention explainer, aiunderstanding.org,
 * "Technical insight").  Visibility follows the flash_attn_func arguments
 * shown on the pages (Workflow 2, Steps 2-3): with `causal`, key j is visible
 * to query i only if j <= i; with window_left = w >= 0, only if j >= i - w;
 * window_left = -1 means no window (the pages' window_size=(-1,-1)); the
 * right entry of window_size, taken by fa_fwd_window / fa_bwd_window, keeps
 * only j <= i + window_right (local attention on both sides).  Query
 * and key indices are absolute (top-left aligned) also when N_q != N_k.  A
 * row that sees no key gets O = 0 and LSE = -inf.
 *
 * Layouts (the pages' flash_attn_func layout [batch, seqlen, nheads,
 * headdim], Workflow 2, Step 2), all contiguous, row-major:
 *     q, out : [B, N_q, H, D]      k, v : [B, N_k, H, D]
 *     lse    : [B, H, N_q] float32 (may be NULL: not written)
 * Element types: FA_FP16 -> q/k/v/out fp16; FA_BF16 -> q/k/v/out bf16;
 * FA_E4M3 -> q/k/v e4m3 (OCP FP8, 1 byte), out bf16.
 *
 * Ownership: the caller allocates and owns every buffer.  The library keeps
 * no pointer after a call returns; its only device memory is a 2 KB pool of
 * work-scheduler counters allocated once per device on the first call there
 * (one pair of counters per stream, left at zero by every launch).
 * Calls are asynchronous on `stream` (NULL = the legacy default stream);
 * outputs are ready when the stream's work completes.  The forward kernel is
 * launched with programmatic stream serialization: it may begin its
 * on-chip prologue while the previous kernel on the stream finishes, and
 * waits for that kernel to complete before it reads or writes any global
 * memory, so stream order holds as for any launch.
 *
 * CUDA graphs: after one call on a stream (which sets kernel attributes and
 * takes the stream's counters), calls on that stream can be captured; a
 * captured forward keeps that stream's counters, so a graph must not be
 * replayed while another forward runs on the stream it was captured on
 * (fa_fwd_noalloc's one fixed array is shared by all its calls likewise).
 *
 * Errors: every entry point returns FA_OK (0) or a negative fa_status and
 * never aborts.  Argument errors are detected before any GPU work is queued.
 * Wait timeouts inside a running kernel are recorded on the device and
 * reported by fa_device_status().
 */
#ifndef FA_B200_H
#define FA_B200_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t / CUstream. */
typedef struct CUstream_st* fa_stream_t;

typedef enum { FA_FP16 = 0, FA_BF16 = 1, FA_E4M3 = 2 } fa_dtype;

typedef enum {
  FA_OK = 0,
  FA_ERR_ARG = -1,         /* bad size, flag, scale or NULL pointer          */
  FA_ERR_UNSUPPORTED = -2, /* head dim / dtype combination not built          */
  FA_ERR_ALIGN = -3,       /* q, k, v or out not 16-byte aligned              */
  FA_ERR_CUDA = -4,        /* CUDA runtime error (no device, launch failure)  */
  FA_ERR_TIMEOUT = -5      /* a kernel wait ran past its limit (see below)    */
} fa_status;

/*
 * fa_fwd -- attention forward for fp16 / bf16 inputs (dtype FA_E4M3 is
 * accepted too and means all descales are 1).
 *   B, H >= 1; N_q, N_k >= 0; D in {64, 128} (FA_E4M3: D = 128).
 *   scale: finite and > 0 (the pages' default is 1/sqrt(D)).
 *   causal: 0 or 1.  window_left: -1 (none) or >= 0.
 * q and out may be NULL when N_q = 0, k and v when N_k = 0 (N_q = 0 is a
 * no-op; N_k = 0 writes O = 0 and LSE = -inf).
 * Returns FA_ERR_ARG / FA_ERR_UNSUPPORTED / FA_ERR_ALIGN without touching
 * the GPU, FA_ERR_CUDA when the launch fails, else FA_OK.
 */
int fa_fwd(const void* q, const void* k, const void* v, void* out, float* lse,
           int B, int N_q, int N_k, int H, int D, float scale, int causal,
           int window_left, int dtype, fa_stream_t stream);

/*
 * fa_fwd_fp8 -- FP8 e4m3 forward with per-tensor scales (the FP8 forward the
 * pages describe for FlashAttention-3, Flash Attention | Hermes Skill,
 * Workflow 3).  The true inputs are q_descale * q, k_descale * k and
 * v_descale * v; out is bf16.  Softmax probabilities are quantised to e4m3
 * (after a power-of-two shift into e4m3's range) for the P*V product; all
 * accumulation is fp32.  Descales must be finite and > 0.
 */
int fa_fwd_fp8(const void* q, const void* k, const void* v, void* out, float* lse,
               int B, int N_q, int N_k, int H, int D, float scale, int causal,
               int window_left, float q_descale, float k_descale, float v_descale,
               fa_stream_t stream);

/*
 * fa_fwd_gqa -- multi-query / grouped-query attention (Flash Attention |
 * Hermes Skill, Workflow 2, Step 3 "Enable advanced features": K and V with
 * fewer heads than Q, shared across query heads).  k and v are
 * [B, N_k, H_kv, D]; q and out [B, N_q, H, D]; H must be a multiple of
 * H_kv >= 1, and query head h reads key/value head h / (H / H_kv)
 * (contiguous groups: the pages do not fix the grouping, this is the
 * plainest reading).  H_kv = 1 is multi-query, H_kv = H the same as
 * fa_fwd / fa_fwd_fp8.  Every other argument, the descales (all 1 for
 * 16-bit inputs) and the return values as for fa_fwd / fa_fwd_fp8.
 */
int fa_fwd_gqa(const void* q, const void* k, const void* v, void* out, float* lse,
               int B, int N_q, int N_k, int H, int H_kv, int D, float scale, int causal,
               int window_left, int dtype, float q_descale, float k_descale, float v_descale,
               fa_stream_t stream);

/*
 * fa_fwd_window -- fa_fwd_gqa with both entries of the pages' window_size
 * (Flash Attention | Hermes Skill, Workflow 2, Step 3: the sliding-window
 * example passes (256, 256), keys on both sides of the query).  Key j is
 * visible to query i only if i - window_left <= j <= i + window_right, -1
 * meaning no bound on that side; causal = 1 still hides every j > i, so a
 * right window beside it changes nothing.  window_right = 0 is causal,
 * window_right >= N_k no right bound.  Every other argument and the return
 * values as fa_fwd_gqa; FA_ERR_ARG also for window_right < -1, or for a right
 * bound with N_q + N_k >= 2^31 - 256.
 */
int fa_fwd_window(const void* q, const void* k, const void* v, void* out, float* lse,
                  int B, int N_q, int N_k, int H, int H_kv, int D, float scale, int causal,
                  int window_left, int window_right, int dtype, float q_descale, float k_descale,
                  float v_descale, fa_stream_t stream);

/*
 * fa_fwd_splitkv -- the forward of fa_fwd_gqa with the key range split into
 * up to num_splits slices that run as separate work units, for shapes with
 * few query tiles and many keys (decode-like N_q << N_k), which would
 * otherwise occupy only B * H * ceil(N_q / 256) of the GPU's SMs.  Every
 * slice computes the same online softmax over its keys and writes its O
 * (normalised by the slice's own row sum) and LSE in fp32 to `workspace`;
 * a second kernel on the same stream combines them:
 *   LSE = log sum_s exp(LSE_s),  O = sum_s exp(LSE_s - LSE) * O_s
 * which is the same softmax over all keys (the explainer page's online
 * softmax rescaling, FlashAttention, aiunderstanding.org, "Technical
 * insight", applied across slices instead of across blocks).
 *   num_splits >= 1; the slices used are min(num_splits, key blocks of 128)
 *   rounded so none is empty; 1 is the plain forward (workspace unused).
 *   workspace: caller-owned device memory of at least
 *   fa_fwd_splitkv_workspace_bytes(...) bytes, 256-byte aligned (NULL
 *   allowed when that size is 0).  The library allocates nothing.
 * Other arguments and return values as fa_fwd_gqa; FA_ERR_ARG also for
 * num_splits < 1 or a missing / short / misaligned workspace.
 */
size_t fa_fwd_splitkv_workspace_bytes(int B, int N_q, int N_k, int H, int D, int num_splits);
int fa_fwd_splitkv(const void* q, const void* k, const void* v, void* out, float* lse,
                   int B, int N_q, int N_k, int H, int H_kv, int D, float scale, int causal,
                   int window_left, int dtype, float q_descale, float k_descale,
                   float v_descale, int num_splits, void* workspace, size_t workspace_bytes,
                   fa_stream_t stream);

/*
 * fa_fwd_mask -- the forward of fa_fwd_gqa with an attention mask, the
 * `attn_mask` of the pages' scaled_dot_product_attention call (Flash
 * Attention | Hermes Skill, Workflow 1, Step 2), read with that call's
 * convention:
 *   FA_MASK_BOOL: bytes, key j takes part for query i where the byte is
 *                 nonzero;
 *   FA_MASK_ADD:  16-bit floats (fp16 for fp16 inputs, else bf16) added to
 *                 the scaled score scale * q_i.k_j before the softmax
 *                 (-inf removes the key).
 * Element (b, h, i, j) is at mask + b * mask_stride_b + h * mask_stride_h
 * + i * mask_stride_q + j (strides in elements; 0 broadcasts over batch or
 * heads).  mask must be 16-byte aligned, mask_stride_q >= N_k, and every
 * stride times the element size a multiple of 16 bytes.  Causal and window
 * visibility apply as well; every key block in their range is computed.
 * A row whose keys are all masked gets O = 0, LSE = -inf.  Other arguments
 * and return values as fa_fwd_gqa; FA_ERR_ARG also for a bad mask type,
 * pointer or stride.
 */
typedef enum { FA_MASK_BOOL = 1, FA_MASK_ADD = 2 } fa_mask_type;
int fa_fwd_mask(const void* q, const void* k, const void* v, void* out, float* lse,
                int B, int N_q, int N_k, int H, int H_kv, int D, float scale, int causal,
                int window_left, int dtype, float q_descale, float k_descale, float v_descale,
                const void* mask, int mask_type, long long mask_stride_b, long long mask_stride_h,
                long long mask_stride_q, fa_stream_t stream);

/*
 * fa_fwd_varlen -- the forward over a packed batch of sequences of different
 * lengths (the pages recommend the library for long sequences and batched
 * inference, Flash Attention | Hermes Skill, "When to use" / "Common
 * issues"; the packed layout is this library's reading).  Sequence b owns
 * query rows [cu_seqlens_q[b], cu_seqlens_q[b+1]) of q and out, and keys
 * [cu_seqlens_k[b], cu_seqlens_k[b+1]) of k and v; attention, causal and
 * window rules apply within each sequence, with indices counted from its
 * first row / key (as fa_fwd does for one batch).
 *   q, out: [total_q, H, D]; k, v: [total_k, H_kv, D] (16-byte aligned,
 *     contiguous; out bf16 for FA_E4M3, else the input type).
 *   lse: [H, total_q] fp32, may be NULL.
 *   cu_seqlens_q, cu_seqlens_k: DEVICE arrays of B + 1 int32, 4-byte
 *     aligned, starting at 0, non-decreasing, ending at total_q / total_k.
 *     The kernels read them and clamp every sequence into [0, total]; values
 *     that break these rules give wrong results, never accesses outside the
 *     tensors.
 *   max_seqlen_q >= every sequence's query count (rows past it are not
 *     computed); max_seqlen_k >= every key count (it sizes the L2 grouping).
 * dtype, descales and the rest as fa_fwd_gqa.  Returns FA_ERR_ARG for bad
 * sizes or pointers (before any GPU work), else as fa_fwd_gqa.
 */
int fa_fwd_varlen(const void* q, const void* k, const void* v, void* out, float* lse,
                  const int* cu_seqlens_q, const int* cu_seqlens_k, int B, int max_seqlen_q,
                  int max_seqlen_k, int total_q, int total_k, int H, int H_kv, int D, float scale,
                  int causal, int window_left, int dtype, float q_descale, float k_descale,
                  float v_descale, fa_stream_t stream);

/*
 * fa_fwd_dropout -- the forward with dropout of the attention probabilities
 * (the dropout_p argument of the pages' flash_attn_func, Flash Attention |
 * Hermes Skill, Workflow 2, Step 2, which gives no definition; this
 * library's reading): after the softmax, each probability P_ij is kept with
 * probability 1 - p and divided by 1 - p, or dropped, independently:
 *     O_i = sum_j (Z_ij / (1 - p)) P_ij V_j,   LSE as without dropout.
 * Z_ij = 1 when the 16-bit value for key j of row i of (batch b, query head
 * h) is >= round(p * 65536) (ties to even; p taken as the float given).
 * The values come from Philox4x32-10 (Salmon et al., "Parallel Random
 * Numbers: As Easy as 1, 2, 3", SC 2011) at counter
 * (j / 8, i, b * H + h, offset) with key (seed mod 2^32, seed / 2^32): the
 * (j mod 2) half (low half first) of output word (j mod 8) / 2.  Calls with
 * the same seed and offset drop the same keys (fa_bwd_dropout needs them);
 * change offset (or seed) for a new mask.
 *   Arguments as fa_fwd_gqa (FA_FP16 / FA_BF16 only) plus dropout_p in
 * [0, 1) (0 = plain forward), seed and offset.  Returns FA_ERR_ARG for p out
 * of range, FA_ERR_UNSUPPORTED for FA_E4M3, else as fa_fwd_gqa.
 */
int fa_fwd_dropout(const void* q, const void* k, const void* v, void* out, float* lse,
                   int B, int N_q, int N_k, int H, int H_kv, int D, float scale, int causal,
                   int window_left, int dtype, float dropout_p, unsigned long long seed,
                   unsigned offset, fa_stream_t stream);

/*
 * fa_fwd_host -- the same forward on HOST buffers: copies q, k, v from host
 * to the caller's device buffers dq, dk, dv, runs fa_fwd / fa_fwd_fp8 into
 * dout / dlse, and copies out (and lse, when both lse and dlse are non-NULL)
 * back to host, all on `stream`.  Host buffers should be pinned for
 * asynchronous copies.  Synchronises `stream` before returning.
 */
int fa_fwd_host(const void* q, const void* k, const void* v, void* out, float* lse,
                void* dq, void* dk, void* dv, void* dout, float* dlse,
                int B, int N_q, int N_k, int H, int D, float scale, int causal,
                int window_left, int dtype, float q_descale, float k_descale,
                float v_descale, fa_stream_t stream);

/*
 * fa_fwd_host_async -- fa_fwd_host without the final synchronisation: the
 * copies in, the forward and the copies out are enqueued on `stream` and the
 * call returns.  out and lse hold the result once `stream` has completed
 * (synchronise it, or wait on an event recorded after the call); the host
 * buffers must stay valid and unmodified until then, and must be pinned for
 * the copies to overlap other work.  Calls on different streams with their
 * own device buffers run concurrently, so one batch's copies in overlap
 * another's forward and copies out.  Arguments and return values as
 * fa_fwd_host.
 */
int fa_fwd_host_async(const void* q, const void* k, const void* v, void* out, float* lse,
                      void* dq, void* dk, void* dv, void* dout, float* dlse,
                      int B, int N_q, int N_k, int H, int D, float scale, int causal,
                      int window_left, int dtype, float q_descale, float k_descale,
                      float v_descale, fa_stream_t stream);

/*
 * fa_fwd_noalloc -- the forward of fa_fwd / fa_fwd_fp8 (dtype FA_E4M3 uses
 * the three descales; other dtypes take 1.0) for callers that cannot
 * allocate device memory: code whose allocations must all come from its own
 * pre-reserved pool or arena, code that must not take the allocator's locks
 * or risk an allocation failure on its launch path, and code running where
 * cudaMalloc is not permitted.  The paper has no counterpart; it is an
 * interface choice of this library.
 *   This call allocates nothing (no cudaMalloc, cudaFree or allocating
 * library routine).  The work scheduler's scratch, two 32-bit counters,
 * lives in a fixed 256-byte device array inside the library, which every GPU
 * that loads the library holds until the process exits.  Its first call on
 * a device looks up that array's device address (once, with the device
 * current); make that first call before any stream capture.  Each call
 * clears the counters on `stream` before its kernel, and the kernel leaves
 * them at zero.  All calls share the one array, so calls that overlap on the
 * GPU (for instance on two streams) race and give wrong results: issue them
 * in order.  Inputs, outputs, layouts and errors are those of fa_fwd;
 * problems with more work units than the 32-bit counters can index are
 * rejected with FA_ERR_ARG.
 */
int fa_fwd_noalloc(const void* q, const void* k, const void* v, void* out, float* lse,
                   int B, int N_q, int N_k, int H, int D, float scale, int causal,
                   int window_left, int dtype, float q_descale, float k_descale,
                   float v_descale, fa_stream_t stream);

/*
 * fa_bwd -- gradients of the forward for FA_FP16 / FA_BF16 inputs (K/V heads
 * equal to query heads): given dout = dL/dO, writes dq = dL/dQ, dk, dv.  The
 * pages give the backward only by its method, recomputation of the attention
 * matrix from the inputs and the forward's softmax statistics (Flash
 * Attention | Hermes Skill, "Quick start"; FlashAttention-3 FP16/BF16
 * forward and backward, "Workflow 3: H100 FP8 optimization
 * (FlashAttention-3)"); the result is the exact vector-Jacobian product of
 * the forward defined above:
 *     P = exp(S - LSE),  dV = P^T dO,  dP = dO V^T,
 *     dS = P * (dP - rowsum(dO * O)),  dQ = scale dS K,  dK = scale dS^T Q.
 *   q, k, v, out, lse: the forward's inputs and outputs (same B, N_q, N_k,
 *     H, D, scale, causal, window_left, dtype); lse is required here.
 *   dout, dq: [B, N_q, H, D]; dk, dv: [B, N_k, H, D]; 16-bit like q.
 *   workspace: caller-owned device memory of at least
 *     fa_bwd_workspace_bytes(B, N_q, H, D) bytes, 256-byte aligned: the fp32
 *     row term rowsum(dO * O), [B, H, N_q].  The library allocates nothing.
 * Three kernels run in order on `stream`: the row term; dK and dV (one CTA
 * per key block); dQ (one CTA per query block).  Returns FA_ERR_ARG /
 * FA_ERR_UNSUPPORTED (FA_E4M3, other head dims) / FA_ERR_ALIGN (16-byte
 * aligned tensors, 4-byte aligned lse) before any GPU work, FA_ERR_CUDA on a
 * launch failure, else FA_OK; waits that time out are reported by
 * fa_device_status().  fa_bwd_workspace_bytes returns 0 for invalid sizes.
 */
size_t fa_bwd_workspace_bytes(int B, int N_q, int H, int D);
int fa_bwd(const void* q, const void* k, const void* v, const void* out, const void* dout,
           const float* lse, void* dq, void* dk, void* dv, int B, int N_q, int N_k, int H, int D,
           float scale, int causal, int window_left, int dtype, void* workspace,
           size_t workspace_bytes, fa_stream_t stream);

/*
 * fa_bwd_gqa -- fa_bwd for grouped K/V heads (the forward of fa_fwd_gqa;
 * multi-query / grouped-query attention, Flash Attention | Hermes Skill,
 * Workflow 2, Step 3): k, v, dk, dv are [B, N_k, H_kv, D] with H a multiple
 * of H_kv, and query head h reads K/V head h / (H / H_kv).  dk and dv of a
 * K/V head are the sums of the gradients of every query head that reads it.
 * Workspace, ownership, kernels and return values as fa_bwd; FA_ERR_ARG also
 * when H_kv < 1 or H is not a multiple of H_kv.
 */
int fa_bwd_gqa(const void* q, const void* k, const void* v, const void* out, const void* dout,
               const float* lse, void* dq, void* dk, void* dv, int B, int N_q, int N_k, int H,
               int H_kv, int D, float scale, int causal, int window_left, int dtype,
               void* workspace, size_t workspace_bytes, fa_stream_t stream);

/*
 * fa_bwd_window -- fa_bwd_gqa for the forward of fa_fwd_window: the same
 * causal, window_left and window_right.  Workspace, ownership, kernels and
 * return values as fa_bwd_gqa; FA_ERR_ARG also as fa_fwd_window.
 */
int fa_bwd_window(const void* q, const void* k, const void* v, const void* out, const void* dout,
                  const float* lse, void* dq, void* dk, void* dv, int B, int N_q, int N_k, int H,
                  int H_kv, int D, float scale, int causal, int window_left, int window_right,
                  int dtype, void* workspace, size_t workspace_bytes, fa_stream_t stream);

/*
 * fa_bwd_varlen -- the backward of fa_fwd_varlen over the same packed batch:
 * q, out, dout, dq [total_q, H, D]; k, v, dk, dv [total_k, H_kv, D]; lse
 * [H, total_q] (the forward's); cu_seqlens_q / cu_seqlens_k, B, causal and
 * window_left as given to the forward.  Gradients are taken within each
 * sequence; keys no query of their sequence sees get dK = dV = 0.  Here
 * max_seqlen_q and max_seqlen_k must bound every sequence's query and key
 * count (the launch covers that many blocks per sequence; rows or keys past
 * them are not computed).  workspace: fa_bwd_workspace_bytes(1, total_q, H,
 * D) bytes, 256-byte aligned.  Returns FA_ERR_ARG for bad sizes or pointers
 * (before any GPU work), else as fa_bwd_gqa.
 */
int fa_bwd_varlen(const void* q, const void* k, const void* v, const void* out, const void* dout,
                  const float* lse, void* dq, void* dk, void* dv, const int* cu_seqlens_q,
                  const int* cu_seqlens_k, int B, int max_seqlen_q, int max_seqlen_k, int total_q,
                  int total_k, int H, int H_kv, int D, float scale, int causal, int window_left,
                  int dtype, void* workspace, size_t workspace_bytes, fa_stream_t stream);

/*
 * fa_bwd_dropout -- fa_bwd_gqa for the forward of fa_fwd_dropout: the same
 * dropout_p, seed and offset redraw the forward's keep bits, and the
 * gradients are those of O = (Z / (1 - p) * P) V: dV = (Z P / (1 - p))^T dO,
 * dP = Z / (1 - p) * (dO V^T), dS = P * (dP - rowsum(dO * O)), dQ, dK as
 * fa_bwd.  out and lse are the dropout forward's.  dropout_p = 0 is fa_bwd_gqa.
 * Workspace, kernels and return values as fa_bwd; FA_ERR_ARG for p outside
 * [0, 1).
 */
int fa_bwd_dropout(const void* q, const void* k, const void* v, const void* out, const void* dout,
                   const float* lse, void* dq, void* dk, void* dv, int B, int N_q, int N_k, int H,
                   int H_kv, int D, float scale, int causal, int window_left, int dtype,
                   float dropout_p, unsigned long long seed, unsigned offset, void* workspace,
                   size_t workspace_bytes, fa_stream_t stream);

/*
 * fa_fwd_ex / fa_bwd_ex -- one call with every option of the pages'
 * flash_attn_func that can be combined (Flash Attention | Hermes Skill,
 * Workflow 2, Steps 2-3: dropout_p, causal, window_size=(left, right),
 * K/V with fewer heads), over a padded or a packed batch.  The fields take
 * the meanings of the entry points above:
 *   q ... lse, B, N_q, N_k, H, H_kv, D, scale, causal, window_left, dtype and
 *     the descales as fa_fwd_gqa; window_right as fa_fwd_window;
 *   cu_seqlens_q / cu_seqlens_k (both NULL: the padded batch [B, N_q / N_k,
 *     ...]; both set: the packed batch of fa_fwd_varlen, B sequences, N_q /
 *     N_k the longest (fa_bwd_ex: every sequence at most that long), total_q
 *     / total_k the packed rows);
 *   dropout_p, seed, offset as fa_fwd_dropout (0 = no dropout; FA_FP16 /
 *     FA_BF16 only); in a packed batch sequence b draws as batch b would.
 * fa_bwd_ex adds out, dout, dq, dk, dv and the workspace of fa_bwd
 * (fa_bwd_workspace_bytes(B, N_q, H, D), or (1, total_q, H, D) for a packed
 * batch) and takes the forward's options unchanged; FA_E4M3 is refused
 * there.  A mask or a split key range is not an option here (fa_fwd_mask,
 * fa_fwd_splitkv).  Validation, ownership and return values as the entry
 * points whose fields they are; FA_ERR_ARG also for a NULL args pointer or
 * only one of the two cu_seqlens pointers.
 */
typedef struct fa_fwd_args {
  const void* q;
  const void* k;
  const void* v;
  void* out;
  float* lse;
  int B, N_q, N_k, H, H_kv, D;
  float scale;
  int causal, window_left, window_right;
  int dtype;
  float q_descale, k_descale, v_descale;
  const int* cu_seqlens_q;
  const int* cu_seqlens_k;
  int total_q, total_k;
  float dropout_p;
  unsigned long long seed;
  unsigned offset;
} fa_fwd_args;

typedef struct fa_bwd_args {
  const void* q;
  const void* k;
  const void* v;
  const void* out;
  const void* dout;
  const float* lse;
  void* dq;
  void* dk;
  void* dv;
  int B, N_q, N_k, H, H_kv, D;
  float scale;
  int causal, window_left, window_right;
  int dtype;
  const int* cu_seqlens_q;
  const int* cu_seqlens_k;
  int total_q, total_k;
  float dropout_p;
  unsigned long long seed;
  unsigned offset;
  void* workspace;
  size_t workspace_bytes;
} fa_bwd_args;

int fa_fwd_ex(const fa_fwd_args* args, fa_stream_t stream);
int fa_bwd_ex(const fa_bwd_args* args, fa_stream_t stream);

/*
 * fa_device_status -- synchronises `stream`, then reads and clears the
 * device status word that kernels set when a wait times out.  Returns FA_OK,
 * FA_ERR_TIMEOUT (and the raw flag bits in *flags when flags != NULL) or
 * FA_ERR_CUDA.
 */
int fa_device_status(fa_stream_t stream, int* flags);

/* Upper bound of every in-kernel wait, in nanoseconds (default 2e9). */
void fa_set_wait_limit_ns(unsigned long long limit_ns);

/*
 * fa_wait_probe -- launches one CTA whose wait nothing completes, with the
 * given limit; used to check that waits end and report FA_ERR_TIMEOUT
 * through fa_device_status instead of hanging.
 */
int fa_wait_probe(unsigned long long limit_ns, fa_stream_t stream);

/*
 * fa_exp2_check -- diagnostic: for the n device floats x, writes 2^x as the
 * FMA-pipe polynomial of the given degree (2 or 3: the forward's; 5: the
 * backward's) takes it into poly, and as the exponential unit's
 * approximation (ex2.approx.ftz) takes it into mufu, both device arrays of
 * n floats.  The polynomial clamps x at
 * -125 (2^x below 2^-124 comes out as about 2^-125).  Runs on `stream`;
 * FA_ERR_ARG for n < 0, another degree or a NULL pointer with n > 0.
 */
int fa_exp2_check(const float* x, float* poly, float* mufu, int n, int degree, fa_stream_t stream);

/* Static description of a status code. */
const char* fa_status_string(int status);

/* Library version, e.g. "0.1.0". */
const char* fa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FA_B200_H */
