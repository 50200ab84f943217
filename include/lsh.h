/*
 * lsh.h — C ABI of the B200 (sm_100a) Reformer LSH self-attention library.
 *
 * The method (sources: "Reformer: The Efficient Transformer", research.elamur.ai
 * summary page — Summary paragraph and Key points "LSH attention",
 * "Shared-QK Transformer", "Number of hash rounds"):
 *   1. queries and keys are one shared vector x per token (shared-QK);
 *   2. each hash round r maps x to a bucket h_r(x) = argmax([x R_r ; -x R_r])
 *      with a random matrix R_r;
 *   3. positions are sorted by bucket, separately for every round;
 *   4. each chunk of m sorted positions attends to itself and the chunk
 *      before it; a token does not attend to itself unless it has no other
 *      valid target;
 *   5. the rounds' outputs are combined by a softmax over their per-round
 *      log-sum-exps; the backward pass recomputes the attention weights.
 *
 * Conventions shared by every entry point
 *   - All tensor arguments are DEVICE pointers, contiguous, row-major, owned
 *     and allocated by the caller. The library allocates no memory while it
 *     runs: scratch space comes from the caller through (ws, ws_bytes),
 *     256-byte aligned, of at least the size the matching *_workspace_size()
 *     returns. Its only device memory is static, held by every GPU that loads
 *     the library until the process exits: a 4-byte status word and the
 *     16 MiB scratch array of lsh_sort_noalloc, whose contents persist from
 *     one lsh_sort_noalloc call to the next.
 *   - Work is queued asynchronously on `stream` (NULL = legacy default
 *     stream). Nothing synchronises unless stated.
 *   - Arguments are checked on the host before anything is launched; a bad
 *     argument returns LSH_ERR_INVALID_ARG / LSH_ERR_UNSUPPORTED /
 *     LSH_ERR_WORKSPACE and launches nothing. A failed launch returns
 *     LSH_ERR_CUDA. Kernels that wait on hardware barriers give up after one
 *     second of waiting and record LSH_ERR_TIMEOUT in a device status word,
 *     read by lsh_device_status(). No C++ exception crosses the ABI.
 *   - bf16 problems with chunk 64 run on the tensor cores, where gathered
 *     rows, attention weights and their gradients pass through fp16 (fp32
 *     accumulation): inputs, outputs and gradients must stay inside the fp16
 *     range (|value| < 65504). This path checks every result it writes
 *     (out, dqk, dv) and records LSH_ERR_RANGE in the device status word when
 *     one is not finite, which is what an input or intermediate outside the
 *     fp16 range produces; such a problem can be run on the CUDA cores by
 *     passing float32 inputs. Other problems run on CUDA cores in fp32.
 *   - Outputs are overwritten, never accumulated into.
 *   - Shapes: B batch, H heads, L sequence length, d head size (64),
 *     n_buckets (even), n_rounds hash rounds, chunk = m.
 *     qk, v, out, out_lo, dout: [B, H, L, d] in `dtype`;
 *     R: [n_rounds, d, n_buckets/2] in `dtype`;
 *     bucket, perm: [B, H, n_rounds, L] int32;
 *     lse: [B, H, L] float32; dqk, dv: [B, H, L, d] float32.
 *   - B*H*L == 0 is a valid empty problem: nothing is launched, LSH_OK.
 */
#ifndef LSH_H
#define LSH_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st* lsh_stream_t;

typedef enum {
  LSH_OK = 0,
  LSH_ERR_INVALID_ARG = 1,   /* null pointer, bad size or bad combination      */
  LSH_ERR_UNSUPPORTED = 2,   /* valid but not implemented (e.g. d != 64)       */
  LSH_ERR_WORKSPACE = 3,     /* workspace missing, too small or misaligned     */
  LSH_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed           */
  LSH_ERR_TIMEOUT = 5,       /* a kernel gave up waiting on a barrier          */
  LSH_ERR_DEVICE_CHECK = 6,  /* a kernel found an out-of-range index           */
  LSH_ERR_RANGE = 7          /* a tensor-core-path result is not finite: an input
                                or intermediate left the fp16 range            */
} lsh_status;

typedef enum { LSH_F32 = 0, LSH_BF16 = 1 } lsh_dtype;

typedef struct {
  int32_t B, H, L, d;
  int32_t n_buckets;   /* even, 2 .. 65536                                     */
  int32_t n_rounds;    /* 1 .. 64                                              */
  int32_t chunk;       /* m: a multiple of 64 that divides L                  */
  int32_t causal;      /* 0: every key in the window; 1: keys at earlier positions only */
  float scale;         /* logit scale, usually 1/sqrt(d)                      */
  int32_t dtype;       /* lsh_dtype of qk, v, R, out, dout                    */
} lsh_problem;

/*
 * lsh_hash — step 2 (Key points, "LSH attention": h(x) = argmax([xR; -xR])).
 *   bucket[b,h,r,i] = argmax over the n_buckets entries of [x R_r ; -x R_r],
 *   x = qk[b,h,i,:], lowest index on exact ties, for every round r.
 *   The contraction accumulates exact products in float32 (bf16 inputs
 *   multiply exactly; float32 inputs use fused multiply-add).
 */
lsh_status lsh_hash(const lsh_problem* p, const void* qk, const void* R,
                    int32_t* bucket, lsh_stream_t stream);

/*
 * lsh_sort — step 3 (Summary and Key points: positions "sorted by bucket").
 *   For every (b,h,r): perm[b,h,r,t] = original position of sorted slot t,
 *   where positions are sorted stably by bucket, i.e. by the packed key
 *   (round, bucket, position). bucket values must lie in [0, n_buckets).
 */
size_t lsh_sort_workspace_size(const lsh_problem* p);
lsh_status lsh_sort(const lsh_problem* p, const int32_t* bucket, int32_t* perm,
                    void* ws, size_t ws_bytes, lsh_stream_t stream);

/*
 * lsh_attn_fwd — steps 4 and 5 (Key points "LSH attention" and
 *   "Shared-QK Transformer"). For each round, the query in sorted slot t
 *   (chunk c = t / m) attends to the keys in slots [max(0,(c-1)m), (c+1)m)
 *   of the same round. Key j is valid for query i iff j != i and, when
 *   causal, j < i (original positions). Logits are scale * x_i . x_j.
 *   Per round: lse_r,i (or -inf with no valid key) and o_r,i; then
 *   lse[i] = log sum_r exp(lse_r,i), out[i] = sum_r exp(lse_r,i - lse[i]) o_r,i.
 *   A token with no valid key in any round attends to itself:
 *   out[i] = v[i], lse[i] = -inf.
 *   out_lo (optional, may be NULL; same shape and dtype as out): for bf16
 *   problems, the rounding residual out_lo = bf16(O - out) of the float32
 *   result O, so that out + out_lo carries O to about 16 significant bits;
 *   lsh_attn_bwd uses it for D = dout . O. Ignored for float32 problems.
 */
size_t lsh_fwd_workspace_size(const lsh_problem* p);
lsh_status lsh_attn_fwd(const lsh_problem* p, const void* qk, const void* v,
                        const int32_t* perm, void* out, void* out_lo, float* lse,
                        void* ws, size_t ws_bytes, lsh_stream_t stream);

/*
 * lsh_attn_bwd — gradient of sum(out * dout) with respect to qk and v,
 *   recomputing the attention weights P_ij = exp(s_ij - lse_i) instead of
 *   storing them (the Reformer's recompute-instead-of-store principle,
 *   Summary paragraph). D_i = dout_i . out_i; dS = P (dout_i . v_j - D_i);
 *   dqk receives scale * dS x from both the query and the key side (keys are
 *   the queries); dv_j += P_ij dout_i; a self-attending token passes dout
 *   to dv. `out`, `out_lo` and `lse` are lsh_attn_fwd's outputs for the same
 *   inputs; out_lo may be NULL, in which case D is formed from `out` alone
 *   (for bf16 problems that adds the rounding error of out to D).
 *   Workspace: D (4 bytes per token) and, for the tensor-core path (bf16,
 *   chunk 64), fp16 copies of qk, v and dout (384 bytes per token), the
 *   per-round fp16 partial gradients in token order (256 bytes per token and
 *   round) and a map of the partial rows at work-unit edges (4 bytes per
 *   token and round). dqk and dv are overwritten, not accumulated into.
 */
size_t lsh_bwd_workspace_size(const lsh_problem* p);
lsh_status lsh_attn_bwd(const lsh_problem* p, const void* qk, const void* v,
                        const int32_t* perm, const void* out, const void* out_lo,
                        const float* lse, const void* dout, float* dqk, float* dv,
                        void* ws, size_t ws_bytes, lsh_stream_t stream);

/*
 * lsh_local_attn_fwd / lsh_local_attn_bwd — local chunked self-attention
 *   ("The Reformer - Pushing the limits of language modeling", Approach and
 *   Takeaways: the input is cut into chunks of length l_c, and each chunk
 *   also sees a configurable overlap of preceding and following chunks).
 *   The queries of chunk c (positions [c m, (c+1) m)) attend to the keys at
 *   positions [max(0, (c - n_back) m), min(L, (c + 1 + n_fwd) m)), with the
 *   same shared-QK self-mask and fall-back, causal mask (j < i) and logit
 *   scale as lsh_attn_fwd, i.e. lsh_attn_fwd's arithmetic in the identity
 *   order with a window of n_back chunks before and n_fwd after.
 *   - p->n_rounds must be 1; p->n_buckets is not used (any valid value).
 *   - 0 <= n_back, n_fwd <= 65536, else LSH_ERR_INVALID_ARG.
 *   - Outputs, out_lo and the backward's gradients as for lsh_attn_fwd /
 *     lsh_attn_bwd; the workspaces come from the *_workspace_size calls with
 *     the same (p, n_back, n_fwd).
 *   - bf16 problems with chunk 64, n_back = 1 and n_fwd = 0 run on the tensor
 *     cores (same fp16 range rule and LSH_ERR_RANGE check as the LSH path);
 *     other problems run on CUDA cores in fp32.
 */
size_t lsh_local_fwd_workspace_size(const lsh_problem* p, int32_t n_back, int32_t n_fwd);
lsh_status lsh_local_attn_fwd(const lsh_problem* p, int32_t n_back, int32_t n_fwd, const void* qk,
                              const void* v, void* out, void* out_lo, float* lse, void* ws,
                              size_t ws_bytes, lsh_stream_t stream);
size_t lsh_local_bwd_workspace_size(const lsh_problem* p, int32_t n_back, int32_t n_fwd);
lsh_status lsh_local_attn_bwd(const lsh_problem* p, int32_t n_back, int32_t n_fwd, const void* qk,
                              const void* v, const void* out, const void* out_lo, const float* lse,
                              const void* dout, float* dqk, float* dv, void* ws, size_t ws_bytes,
                              lsh_stream_t stream);

/*
 * The layer around the attention: a chunked position-wise feed-forward and
 * the reversible residual block ("Reformer: The Efficient Transformer",
 * research.elamur.ai summary page, Key points, "Reversible layers":
 * reversible residual layers (Gomez et al. 2017) recompute a layer's inputs
 * from its outputs in the backward pass instead of storing them; the
 * feed-forward runs in chunks, which leaves its results unchanged).
 *   G(x) = max(0, x W1 + b1) W2 + b2, applied to every position;
 *   F(x2) = lsh_attn_fwd's output with qk = v = x2 (shared-QK attention whose
 *           values are its input; projection weights are not part of this);
 *   forward  y1 = x1 + F(x2), y2 = x2 + G(y1);
 *   backward x2 = y2 - G(y1), x1 = y1 - F(x2), from the outputs alone.
 * Activations x, x1, x2, y, y1, y2 and their gradients are [B, H, L, 64]
 * bf16, the attention's layout: token (b, l) has d_model = 64 H features, its
 * H head rows side by side. W1 [d_model, d_ff] and W2 [d_ff, d_model] are
 * bf16 row-major; b1 [d_ff], b2 [d_model] and all weight gradients are
 * float32. Products run on the tensor cores with float32 accumulation; the
 * hidden activations and their gradient are rounded to bf16 per chunk.
 * Every result is deterministic, and every per-position result (y, dx, the
 * reconstruction) is bit-identical for any ff_chunk.
 */
typedef struct {
  int32_t B, H, L;     /* activations [B, H, L, 64]; L a multiple of 128       */
  int32_t d_ff;        /* hidden width: a multiple of 128, up to 65536         */
  int32_t ff_chunk;    /* positions per feed-forward chunk: a multiple of 128 */
} lsh_ff_problem;

/* y = res + G(x) (res may be NULL: y = G(x)); y may not alias x. */
size_t lsh_ff_workspace_size(const lsh_ff_problem* f);
lsh_status lsh_ff_fwd(const lsh_ff_problem* f, const void* x, const void* W1, const float* b1,
                      const void* W2, const float* b2, const void* res, void* y, void* ws,
                      size_t ws_bytes, lsh_stream_t stream);
/* Backward of y = res + G(x) for the incoming gradient dy:
 *   dx = dres + (dG/dx)^T dy (dres may be NULL), bf16;
 *   dW1, db1, dW2, db2 = gradients of sum(G(x) * dy), overwritten;
 *   rec (optional): y_in - G(x), the reversible block's reconstruction of the
 *   residual branch from its output y_in (both NULL, or both given).
 * The workspace is that of lsh_ff_fwd. */
lsh_status lsh_ff_bwd(const lsh_ff_problem* f, const void* x, const void* W1, const float* b1,
                      const void* W2, const float* b2, const void* dy, const void* dres,
                      const void* y_in, void* rec, void* dx, float* dW1, float* db1, float* dW2,
                      float* db2, void* ws, size_t ws_bytes, lsh_stream_t stream);

/* Reversible block forward: hashes x2 with R, sorts (perm, [B, H, n_rounds,
 * L], is written for the backward), y1 = x1 + F(x2), y2 = x2 + G(y1).
 * p describes the attention (bf16, d 64, same B, H, L as f). */
size_t lsh_rev_fwd_workspace_size(const lsh_problem* p, const lsh_ff_problem* f);
lsh_status lsh_rev_fwd(const lsh_problem* p, const lsh_ff_problem* f, const void* x1,
                       const void* x2, const void* R, const void* W1, const float* b1,
                       const void* W2, const float* b2, void* y1, void* y2, int32_t* perm,
                       void* ws, size_t ws_bytes, lsh_stream_t stream);
/* Reversible block backward from (y1, y2), the incoming gradients (dy1, dy2)
 * and the forward's perm (kept, because a bucket id is a discrete function of
 * x2 and the reconstruction recovers x2 only up to rounding): writes the
 * reconstructed inputs x1, x2, their gradients dx1, dx2 (bf16) and the
 * feed-forward's weight gradients (float32, overwritten). */
size_t lsh_rev_bwd_workspace_size(const lsh_problem* p, const lsh_ff_problem* f);
lsh_status lsh_rev_bwd(const lsh_problem* p, const lsh_ff_problem* f, const void* y1,
                       const void* y2, const void* dy1, const void* dy2, const int32_t* perm,
                       const void* W1, const float* b1, const void* W2, const float* b2,
                       void* x1, void* x2, void* dx1, void* dx2, float* dW1, float* db1,
                       float* dW2, float* db2, void* ws, size_t ws_bytes, lsh_stream_t stream);

/*
 * lsh_sort_noalloc — lsh_sort without a caller workspace. The reference pages
 *   have no counterpart: this entry point exists for callers that cannot
 *   obtain device memory for a workspace, such as a host framework that owns
 *   every byte of device memory and gives kernel libraries no allocation hook,
 *   or a latency-critical loop where cudaMalloc's implicit device-wide
 *   synchronisation is not acceptable. It allocates nothing: its scratch is
 *   one array of LSH_SORT_NOALLOC_SCRATCH_BYTES (16 MiB) in the library's own
 *   device memory, which every GPU that loads the library holds until the
 *   process exits.
 *   - Same arguments, result and checks as lsh_sort. A problem whose
 *     lsh_sort_workspace_size() exceeds the scratch returns LSH_ERR_WORKSPACE
 *     and launches nothing. (16 MiB covers, e.g., 8 heads x 4 rounds x 2^20
 *     positions with 1024 buckets, or 2 x 524288 positions with 8192.)
 *   - All calls on a device share the one scratch array and it keeps the last
 *     call's contents; the sort clears what must start at zero itself. Calls
 *     whose work overlaps on the GPU (other streams, other host threads)
 *     race on the scratch and give wrong results: serialise them.
 *   - The first call on each device looks up the scratch's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture.
 */
#define LSH_SORT_NOALLOC_SCRATCH_BYTES (16u * 1024u * 1024u)
lsh_status lsh_sort_noalloc(const lsh_problem* p, const int32_t* bucket, int32_t* perm,
                            lsh_stream_t stream);

/*
 * lsh_check_wait_timeout — a health check of the failure detection; the
 *   pages have no counterpart. Launches one small kernel in which a single
 *   thread waits, through the same bounded-wait routine as the tensor-core
 *   kernels' pipeline barriers, on a shared-memory barrier that nothing ever
 *   completes. After `limit_ns` nanoseconds of GPU global time (1 .. 1e9) the
 *   wait gives up, LSH_ERR_TIMEOUT is recorded in the device status word
 *   (unless an earlier error is there) and the kernel returns, leaving the
 *   context usable. Read the result with lsh_device_status(). Returns
 *   LSH_ERR_INVALID_ARG for a limit outside that range, LSH_ERR_CUDA if the
 *   launch fails.
 */
lsh_status lsh_check_wait_timeout(uint64_t limit_ns, lsh_stream_t stream);

/* Synchronises `stream`, returns and clears the current device's status
 * word: LSH_OK, or the FIRST error a kernel recorded since the last read
 * (LSH_ERR_TIMEOUT, LSH_ERR_DEVICE_CHECK or LSH_ERR_RANGE). */
lsh_status lsh_device_status(lsh_stream_t stream);

/* Static, NUL-terminated description of a status code. */
const char* lsh_status_string(lsh_status s);

/* Number of kernels this library has launched in this process (a host-side
 * counter, for accounting; never reset). */
uint64_t lsh_launch_count(void);

#ifdef __cplusplus
}
#endif
#endif /* LSH_H */
