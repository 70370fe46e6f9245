/*
 * causalattn.h -- C ABI of libcausalattn: multi-head causal scaled-dot-product
 * self-attention, forward and backward, on NVIDIA B200 (sm_100a).
 *
 * The operation.  For every batch b and head h, with Q, K, V, dO slices of
 * shape [T, d]:
 *     S   = scale * Q K^T                      (scale is normally 1/sqrt(d))
 *     S_ij = -inf  where j > i                 (causal mask, diagonal kept)
 *     P   = softmax(S) along each row
 *     O   = P V,      LSE_i = log sum_j exp(S_ij)   (natural log)
 * as written in "Stanford CS336 walkthrough" (lmnt.cn), section 5.1 model.py,
 * CausalSelfAttention.forward (q @ k^T * 1/sqrt(k.size(-1)), masked_fill of
 * the upper triangle with -inf, softmax, att @ v), section 3.3 of the same
 * page (masked positions get weight 0 after the softmax), and the
 * torch.tril(ones) mask buffer of "Train Your Own LLM from Scratch"
 * (fishgap.com), section 1, which keeps the diagonal.  Attention dropout is
 * the identity (p = 0.0 in every configuration the pages print).
 *
 * The backward is the gradient of that forward for loss.backward() (CS336
 * walkthrough, section 5.2 train.py):
 *     dV = P^T dO,  dP = dO V^T,  delta_i = sum_c dO_ic O_ic,
 *     dS = P o (dP - delta),  dQ = scale dS K,  dK = scale dS^T Q.
 *
 * Document mask (optional).  BOS-aligned best-fit packing puts several
 * documents in one row ("How to build an LLM by hand", agmtopy.github.io,
 * section 5.5).  Reading: a token attends only to earlier tokens of its own
 * document.  doc_offsets is an int32 device array [B, T]; entry [b, i] is the
 * first position of the document that holds position i.  Position i attends
 * to j iff doc_offsets[b, i] <= j <= i.  Valid arrays have doc_offsets[b,0] =
 * 0 and each entry equal to i (a new document) or to the previous entry.
 * NULL means plain causal attention.
 *
 * Layouts.  q, k, v, o, dout, dq, dk, dv: contiguous bf16 [B, H, T, d]
 * (d fastest), the layout of the pages' .view(B, T, H, C//H).transpose(1, 2).
 * lse, delta: contiguous fp32 [B, H, T].
 *
 * Ownership.  Every pointer is caller-owned DEVICE memory on the current CUDA
 * device (its primary context, which the first call on each host thread binds
 * to that thread if nothing has yet).  The library allocates no memory; it keeps no state besides
 * per-device attribute and occupancy caches, one device-side status word and
 * the fixed delta scratch of gpt_attn_bwd_static_ws.
 *
 * Asynchrony.  Calls validate their arguments, enqueue kernels on `stream`
 * (a cudaStream_t; NULL = the legacy default stream) and return.  Outputs are
 * valid once the stream has reached that point.  Inputs are not modified
 * (except where a caller passes an input buffer as the output of a call that
 * allows it: the RoPE + QK-norm calls work in place).
 * dq, dk, dv, o, lse, delta are fully overwritten, never accumulated into.
 *
 * Errors.  Every call returns a gpt_attn_status.  Nothing aborts, throws or
 * exits across this boundary.  Arguments are checked before any CUDA call, so
 * argument errors are reported even on a machine without a GPU.  A launch
 * failure returns GPT_ATTN_ERR_LAUNCH.  Kernels never wait without bound: a
 * wait that exceeds its limit (2 s) makes the kernel record the event in the
 * device status word (read it with gpt_attn_device_status) and exit early,
 * leaving the outputs unspecified.  An invalid doc_offsets array yields
 * unspecified output values but never an out-of-bounds access.
 *
 * Limits.  d in {32, 64, 128}; T >= 1 (any T: tiles past T are masked);
 * B, H >= 1 with B*H*T*d < 2^31 elements per tensor; scale finite and > 0;
 * the bf16 tensors 16-byte aligned, lse/delta/doc_offsets 4-byte aligned.
 */
#ifndef CAUSALATTN_H
#define CAUSALATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define GPT_ATTN_ABI_VERSION 1

typedef enum {
  GPT_ATTN_OK = 0,
  GPT_ATTN_ERR_NULL_PTR = 1,              /* a required pointer is NULL */
  GPT_ATTN_ERR_BAD_SHAPE = 2,             /* B, H or T < 1 */
  GPT_ATTN_ERR_UNSUPPORTED_HEAD_DIM = 3,  /* d not in {32, 64, 128} */
  GPT_ATTN_ERR_MISALIGNED = 4,            /* a pointer breaks the alignment rule above */
  GPT_ATTN_ERR_BAD_DOC_OFFSETS = 5,       /* gpt_attn_check_doc_offsets found an invalid entry */
  GPT_ATTN_ERR_NO_DEVICE = 6,             /* no usable CUDA device */
  GPT_ATTN_ERR_UNSUPPORTED_ARCH = 7,      /* current device is not sm_100 (B200) */
  GPT_ATTN_ERR_LAUNCH = 8,                /* a CUDA call or kernel launch failed */
  GPT_ATTN_ERR_DEVICE_TIMEOUT = 9,        /* a kernel gave up on a bounded wait */
  GPT_ATTN_ERR_NOT_IMPLEMENTED = 10,
  GPT_ATTN_ERR_BAD_SCALE = 11,            /* scale not finite or <= 0 */
  GPT_ATTN_ERR_TOO_LARGE = 12,            /* a tensor exceeds 2^31 - 1 elements */
  GPT_ATTN_ERR_BAD_PARAM = 13             /* rope_base, gain, eps or an FP8 descale out of range */
} gpt_attn_status;

/*
 * Forward.  Reads q, k, v [B,H,T,d]; writes o [B,H,T,d] and lse [B,H,T].
 */
int gpt_attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                 int T, int d, float scale, const int32_t* doc_offsets, void* stream);

/*
 * Backward.  Reads q, k, v, o, dout [B,H,T,d] and lse [B,H,T] (the forward's
 * outputs); writes dq, dk, dv [B,H,T,d].  delta_ws is a caller-provided fp32
 * [B,H,T] workspace that receives delta = rowsum(dout o o).  Equivalent to
 * gpt_attn_bwd_dq_delta (which computes delta into delta_ws), then
 * gpt_attn_bwd_dkdv.
 */
int gpt_attn_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
                 const float* lse, void* dq, void* dk, void* dv, float* delta_ws, int B, int H,
                 int T, int d, float scale, const int32_t* doc_offsets, void* stream);

/*
 * Sliding-window variants.  "How to build an LLM by hand" (agmtopy.github.io),
 * section 9 (the gpt.py walkthrough), lists sliding-window attention among the
 * model's attention features without defining it.  Reading: a window of
 * `window` keys, the query's own position included: position i attends to j
 * iff i - window < j <= i, and, with doc_offsets, also doc_offsets[b,i] <= j.
 * window <= 0 or window >= T is plain (document-)causal attention, identical
 * to gpt_attn_fwd / gpt_attn_bwd.  Everything else (layouts, ownership,
 * asynchrony, errors, limits) is as for those calls; the backward must be
 * given the same window as the forward that produced o and lse.
 */
int gpt_attn_fwd_window(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                        int H, int T, int d, float scale, const int32_t* doc_offsets, int window,
                        void* stream);

int gpt_attn_bwd_window(const void* q, const void* k, const void* v, const void* o,
                        const void* dout, const float* lse, void* dq, void* dk, void* dv,
                        float* delta_ws, int B, int H, int T, int d, float scale,
                        const int32_t* doc_offsets, int window, void* stream);

/*
 * FP8 (e4m3) forward.  "How to build an LLM by hand" (agmtopy.github.io),
 * section 5, item 4: the in-house FP8 training runs the forward matmuls with
 * e4m3 operands through torch._scaled_mm, one fixed scale per tensor (the page
 * notes that dynamic scaling is missing).  Reading for this forward: q8, k8, v8
 * hold e4m3 codes (OCP E4M3: bias 7, no infinities, largest finite 448) of
 * layout [B,H,T,d], one byte per element, standing for descale_q * q8,
 * descale_k * k8, descale_v * v8.  Both products of the attention take e4m3
 * operands, so the attention weights are rounded to e4m3 too:
 *     S  = scale * descale_q * descale_k * Q8 K8^T   (fp32 accumulation)
 *     r  = exp(S - rowmax S)                          (masks as for gpt_attn_fwd)
 *     W8 = e4m3(2^8 * r)                              (round to nearest even)
 *     o  = descale_v * (W8 V8) / rowsum(W8)           (bf16 [B,H,T,d])
 *     lse = rowmax S + log rowsum(r)                  (fp32 [B,H,T], natural log)
 * The weights are rounded relative to each row's final maximum (the kernel
 * makes two passes over the keys).  o therefore differs from the exact
 * attention of the dequantised inputs by at most
 *     sum_j e_j |v_j - o_exact| / (sum_j r_j - sum_j e_j),
 *     e_j = (2^-4 + 2^-14) r_j + 2^-18,
 * plus bf16 rounding of o.  Causal or document-causal (doc_offsets) masks; no
 * window.  descale_q, descale_k, descale_v must be finite and > 0
 * (GPT_ATTN_ERR_BAD_PARAM otherwise); q8, k8, v8 and o 16-byte aligned.
 * Ownership, asynchrony and errors as for gpt_attn_fwd.
 */
int gpt_attn_fwd_fp8(const void* q8, const void* k8, const void* v8, float descale_q,
                     float descale_k, float descale_v, void* o, float* lse, int B, int H, int T,
                     int d, float scale, const int32_t* doc_offsets, void* stream);

/*
 * KV-cache decode.  Generation appends Tq new tokens to a cache of L keys and
 * values (the pages' inference engine keeps a KV cache and attends from the
 * new tokens with FlashAttention-3's kv-cache call on (B, T, H, D) tensors:
 * "How to build an LLM by hand", agmtopy.github.io, section 2).  New token t
 * (0 <= t < Tq) sits at position L - Tq + t and attends to cache positions
 * 0 .. L - Tq + t: the causal rule above, for the last Tq rows.
 *   q:          bf16 [B, Tq, H, d]   (the new tokens' queries)
 *   k_cache,
 *   v_cache:    bf16 [B, L, H, d]    (positions 0 .. L-1, the new tokens' last)
 *   o:          bf16 [B, Tq, H, d];  lse: fp32 [B, H, Tq] (natural log)
 *   workspace:  caller-owned device memory of at least
 *               gpt_attn_decode_workspace_size(B, H, Tq, L, d) bytes, 16-byte
 *               aligned; its contents on entry do not matter.
 * Limits: 1 <= Tq <= 16, Tq <= L, B and H <= 65535, B*L*H*d < 2^31.  Fails
 * with GPT_ATTN_ERR_BAD_SHAPE for a too-small workspace.  Layout, ownership,
 * asynchrony and error rules as above.  Split over 128-key chunks of the cache
 * (one new token: CUDA cores; two or more: tensor cores) and merged in chunk
 * order: the result is deterministic.
 */
size_t gpt_attn_decode_workspace_size(int B, int H, int Tq, int L, int d);

int gpt_attn_decode(const void* q, const void* k_cache, const void* v_cache, void* o, float* lse,
                    void* workspace, size_t workspace_bytes, int B, int H, int Tq, int L, int d,
                    float scale, void* stream);

/*
 * RoPE + QK-norm prologue.  "How to build an LLM by hand" (agmtopy.github.io),
 * section 9 (the gpt.py walkthrough): the attention applies RoPE and then QK
 * Norm ("x1.2") to the queries and keys; the page gives no formulas.  Reading,
 * per row x = q[b,h,t,:] or k[b,h,t,:] (t is the row's position, 0 .. T-1):
 *   u_p       =  x_p cos(t th_p) + x_{p+d/2} sin(t th_p)      (p < d/2)
 *   u_{p+d/2} = -x_p sin(t th_p) + x_{p+d/2} cos(t th_p),  th_p = rope_base^(-2p/d)
 *   out       = gain * u / sqrt(mean(u^2) + eps)
 * (RMS norm without learned weights; the page's x1.2 is `gain`.)  Q and K are
 * processed in one launch.
 *   q, k:          bf16 [B,H,T,d], read
 *   q_out, k_out:  bf16 [B,H,T,d], written; may equal q / k (in place), must not
 *                  otherwise overlap any argument.
 * rope_base finite and > 0, gain finite, eps finite and >= 0, else
 * GPT_ATTN_ERR_BAD_PARAM; eps = 0 on an all-zero row gives NaN, as the formula
 * does.  Layout, ownership, alignment, asynchrony and errors as above.
 */
int gpt_attn_rope_qknorm_fwd(const void* q, const void* k, void* q_out, void* k_out, int B, int H,
                             int T, int d, float rope_base, float gain, float eps, void* stream);

/*
 * Its backward: from q, k (the prologue's INPUTS) and dq_out, dk_out (gradients
 * of the loss with respect to q_out, k_out), writes dq, dk (gradients with
 * respect to q, k):  du = (gain/r) (dz - u <u,dz> / (d r^2)),  dx = RoPE^T du,
 * r = sqrt(mean(u^2) + eps).  dq may equal dq_out and dk may equal dk_out (in
 * place); no other overlap.  Parameters and errors as for the forward.
 */
int gpt_attn_rope_qknorm_bwd(const void* q, const void* k, const void* dq_out, const void* dk_out,
                             void* dq, void* dk, int B, int H, int T, int d, float rope_base,
                             float gain, float eps, void* stream);

/* Backward step 1: delta[b,h,i] = sum_c dout[b,h,i,c] * o[b,h,i,c] (fp32). */
int gpt_attn_bwd_preprocess(const void* o, const void* dout, float* delta, int B, int H, int T,
                            int d, void* stream);

/* Backward step 2: dk, dv [B,H,T,d] from q, k, v, dout, lse and delta. */
int gpt_attn_bwd_dkdv(const void* q, const void* k, const void* v, const void* dout,
                      const float* lse, const float* delta, void* dk, void* dv, int B, int H,
                      int T, int d, float scale, const int32_t* doc_offsets, void* stream);

/*
 * Backward step 3, without a separate delta step: dq [B,H,T,d] from q, k, v,
 * dout and lse, computing delta = rowsum(dout o o) from o and dout on the way
 * and writing it to delta_out (fp32 [B,H,T]) for gpt_attn_bwd_dkdv.  Same
 * result as gpt_attn_bwd_preprocess followed by gpt_attn_bwd_dq.
 */
int gpt_attn_bwd_dq_delta(const void* q, const void* k, const void* v, const void* o,
                          const void* dout, const float* lse, float* delta_out, void* dq, int B,
                          int H, int T, int d, float scale, const int32_t* doc_offsets,
                          void* stream);

/* Backward step 3: dq [B,H,T,d] from q, k, v, dout, lse and delta. */
int gpt_attn_bwd_dq(const void* q, const void* k, const void* v, const void* dout,
                    const float* lse, const float* delta, void* dq, int B, int H, int T, int d,
                    float scale, const int32_t* doc_offsets, void* stream);

/*
 * Backward for callers that cannot allocate device memory -- code running
 * under a framework's caching allocator that owns the whole device, inside a
 * plugin host that lends out only its own tensors, or in a real-time loop
 * where allocation is forbidden, so that no workspace can be created.  Same
 * arguments and results as gpt_attn_bwd minus delta_ws: the delta workspace
 * is a file-scope device array inside the library,
 * GPT_ATTN_STATIC_WS_MAX_ROWS floats (4 MiB), which every GPU that loads the
 * library holds until the process exits.  (The pages have no counterpart to
 * this entry point; it only changes where the scratch lives.)
 *   - Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 *   - Returns GPT_ATTN_ERR_TOO_LARGE when B*H*T > GPT_ATTN_STATIC_WS_MAX_ROWS.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture.
 *   - The array is part of the library's device code: it is reserved when
 *     that code is loaded onto a device, which (with CUDA's default lazy
 *     module loading) happens during the first library call of any kind on
 *     that device -- possibly this one.  A caller whose allocator will own
 *     every free byte of the device should make one library call (any entry
 *     point) or set CUDA_MODULE_LOADING=EAGER before handing the device over;
 *     after that, calls reserve nothing further.
 *   - All calls share the one array, which keeps the last call's contents
 *     (delta is rewritten in full by every call, so nothing needs clearing):
 *     calls whose work overlaps on the GPU -- two streams, two threads --
 *     race on it and must be serialised by the caller.
 */
#define GPT_ATTN_STATIC_WS_MAX_ROWS (1L << 20)
int gpt_attn_bwd_static_ws(const void* q, const void* k, const void* v, const void* o,
                           const void* dout, const float* lse, void* dq, void* dk, void* dv,
                           int B, int H, int T, int d, float scale, const int32_t* doc_offsets,
                           void* stream);

/*
 * Checks a doc_offsets array on the device against the validity rule above.
 * Synchronises `stream`.  Returns GPT_ATTN_OK or GPT_ATTN_ERR_BAD_DOC_OFFSETS.
 * The verdict passes through one library-owned device word per device; calls
 * are serialised inside the library (each clears the word, runs the check and
 * reads the word back before the next may start), so concurrent calls from
 * several threads or streams each get their own array's verdict.
 */
int gpt_attn_check_doc_offsets(const int32_t* doc_offsets, int B, int T, void* stream);

/*
 * Reads (and, if clear != 0, resets) the device status word of the current
 * device: 0 when no kernel has reported a problem.  Bit 31 plus one bit per
 * wait site: a kernel gave up on a bounded wait.  Bit 30: a kernel found its
 * shared-memory layout larger than the dynamic shared memory it was given
 * (after rounding the base up to 1 KB) and returned without computing.  Synchronises the device.  Returns GPT_ATTN_OK, or an
 * error status if the device cannot be read.
 */
int gpt_attn_device_status(unsigned int* out, int clear);

/*
 * Failure-detection self-test: launches one kernel that waits, with the given
 * limit in nanoseconds, on a barrier nothing ever signals.  The kernel must
 * give up, record the timeout and exit.  Synchronises `stream`, clears the
 * status word again and returns GPT_ATTN_ERR_DEVICE_TIMEOUT when the timeout
 * was detected and reported (the expected outcome), GPT_ATTN_OK if it was not.
 */
int gpt_attn_selftest_wait_timeout(uint64_t limit_ns, void* stream);

/* Human-readable name of a status code (static string, never NULL). */
const char* gpt_attn_strerror(int status);

/* GPT_ATTN_ABI_VERSION of the loaded library. */
int gpt_attn_version(void);

/*
 * Text of the CUDA error behind the most recent GPT_ATTN_ERR_LAUNCH returned on
 * the calling thread ("no error" if none).  Static string, never NULL.
 */
const char* gpt_attn_last_cuda_error(void);

#ifdef __cplusplus
}
#endif

#endif /* CAUSALATTN_H */
