/*
 * lact.h -- C ABI of the B200 (sm_100a) LaCT fast-weight TTT layer (forward
 * and backward) and of the block's sliding-window attention.
 *
 * The layer (Large-Chunk Test-Time Training).  Sources are cited by page
 * title and section:
 *   [P1] "LaCT架构核心思想解析" (gsyq.cn) §1.1, §1.2, §2.1, §2.2, §3.2
 *   [P2] "大块测试时训练（LaCT）技术解析" (dpshk.com) §2.1, §2.2.1, §2.2.2
 *   [P3] "LaCT：以大分块更新人工智能的临时记忆" (iplexlaw.co.kr), sections
 *        「局部注意力与非线性记忆相互补充」, 「更新顺序必须遵守信息可见范围」 and
 *        「视频实验和分布式计算」
 *
 * Per (batch b, head h) the layer keeps a SwiGLU fast-weight net
 *     f_W(x) = W2 (silu(W1 x) * (W3 x)),   W1, W3: [dh, d],  W2: [d, dh]
 * ([P3] three-matrix SwiGLU memory; [P1 §1.2] shapes).  Queries and keys are
 * first mapped to silu(x)/||silu(x)|| over the head dim ([P1 §1.2]).  The
 * sequence is cut into chunks of `chunk` tokens (the last one may be
 * shorter).  For each chunk c:
 *   apply   o_t = f_W(q_t) for the chunk's queries ([P2 §2.1], eq. 2);
 *   update  G_j = d/dW_j [ -sum_{i in c} lr[i,j] <f_W(k_i), v_i> ]
 *           (chunk-summed, per-token rates; j = 0: W1, 1: W2, 2: W3;
 *           [P2 §2.1] eqs. 4-5, [P3]), then a rule
 *             GD:        U = G
 *             momentum:  M <- mean_{i in c}(beta_i) M + G, U = M   [P1 §1.2]
 *             Muon:      U = NewtonSchulz5(G / (||G||_F + 1e-7)),
 *                        quintic (3.4445, -4.7750, 2.0315)         [P2 §2.2.1]
 *           and W_j <- W_j - U_j with every row of W_j scaled back to its
 *           norm before the update ([P2 §2.2.1] eq. 8; rows of W1/W3 have
 *           length d, rows of W2 length dh).
 * Order ([P3] 「更新顺序…」, [P1 §2.2]): LACT_APPLY_THEN_UPDATE (causal
 * sequences: chunk c reads the state left by chunks < c) or
 * LACT_UPDATE_THEN_APPLY (sets: chunk c reads the state after itself).
 *
 * Memory: every pointer passed to lact_ttt_fwd is a DEVICE pointer owned by
 * the caller; the library allocates nothing.  Calls are asynchronous on the
 * caller's CUDA stream (`stream` is a cudaStream_t, NULL = legacy default).
 * Layouts (all dense, row-major, no padding):
 *   q      [B, H, Tq, d]  dtype        raw queries (the prologue runs inside)
 *   k, v   [B, H, T, d]   dtype        raw keys, values
 *   lr     [B, H, T, 3]   float32      per-token rates, already softplus-ed,
 *                                      columns (W1, W2, W3)
 *   beta   [B, H, T]      float32      per-token momentum, already sigmoid-ed;
 *                                      read only when rule == MOMENTUM
 *   w1, w3 [Hw, dh, d]    float32      initial fast weights, Hw = H (shared
 *   w2     [Hw, d, dh]    float32        by the batch, w_shared = 1) or B*H
 *   out    [B, H, Tq, d]  dtype        layer output
 *   w1_out, w3_out [B*H, dh, d], w2_out [B*H, d, dh]  float32  final state;
 *          each may alias the matching input exactly (in-place update,
 *          only when w_shared = 0); any other overlap is rejected.
 *   dtype = LACT_F32 (fp32 path, SIMT kernels) or LACT_BF16 (bf16 tensor-core
 *   path; fp32 fast-weight masters, fp32 accumulation).
 * Alignment: all device pointers 16-byte aligned.
 * Limits: 1 <= d <= 512, 1 <= dh <= 4096 (bf16 path: both multiples of 64);
 *   B*H <= 4096; 1 <= T, Tq <= 2^30; chunk >= 1 (a chunk >= T means one
 *   chunk); Tq == T unless there is a single chunk.
 *
 * Errors: every entry point returns LACT_OK (0) or a negative code.  Argument
 * errors (LACT_EINVAL, LACT_ENOSPC) are found before anything is enqueued.
 * LACT_ECUDA means a launch failed part way; the outputs are then undefined.
 * Device-side failures (a bounded wait inside a kernel that gave up) are
 * recorded in a device status word and reported by lact_ttt_status().
 */
#ifndef LACT_H
#define LACT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum {
  LACT_OK = 0,
  LACT_EINVAL = -1,       /* bad shape, dtype, order, rule, null or misaligned
                             pointer, partial aliasing, unsupported size */
  LACT_ENOSPC = -2,       /* workspace smaller than lact_ttt_workspace_bytes() */
  LACT_ECUDA = -3,        /* a CUDA runtime call or kernel launch failed */
  LACT_ETIMEOUT = -4,     /* a bounded device wait gave up (see lact_ttt_status) */
  LACT_ENODEV = -5,       /* the current device is not an sm_100 GPU */
  LACT_ETOOBIG = -6,      /* the problem needs more scratch than the built-in
                             buffer of lact_ttt_fwd_noalloc holds */
  LACT_ECOMM = -7         /* the context-parallel all-reduce hook failed */
};

enum { LACT_F32 = 0, LACT_BF16 = 1 };
enum { LACT_APPLY_THEN_UPDATE = 0, LACT_UPDATE_THEN_APPLY = 1 };
enum { LACT_RULE_GD = 0, LACT_RULE_MOMENTUM = 1, LACT_RULE_MUON = 2 };

/* Problem description shared by every entry point. */
typedef struct lact_problem {
  int64_t B, H;     /* batch, heads */
  int64_t T;        /* key/value tokens per (b, h) */
  int64_t Tq;       /* query tokens per (b, h) */
  int64_t d, dh;    /* head dim, fast-net hidden dim */
  int64_t chunk;    /* tokens per update (the last chunk may be shorter) */
  int32_t order;    /* LACT_APPLY_THEN_UPDATE or LACT_UPDATE_THEN_APPLY */
  int32_t rule;     /* LACT_RULE_GD, LACT_RULE_MOMENTUM or LACT_RULE_MUON */
  int32_t dtype;    /* LACT_F32 or LACT_BF16: q, k, v and out */
  int32_t w_shared; /* 1: w1/w2/w3 hold H states shared over the batch; 0: B*H */
} lact_problem;

/* Device scratch bytes lact_ttt_fwd needs for problem *p (0 if *p is invalid).
 * Pure host arithmetic; needs no GPU. */
size_t lact_ttt_workspace_bytes(const lact_problem* p);

/* The layer forward, enqueued on `stream`.  All tensor pointers are device
 * pointers in the layouts above; `workspace` is device scratch of at least
 * lact_ttt_workspace_bytes(p) bytes, 256-byte aligned, owned by the caller
 * and not touched by anything else until the stream reaches the end of this
 * call.  beta may be NULL unless rule == LACT_RULE_MOMENTUM. */
int lact_ttt_fwd(const lact_problem* p,
                 const void* q, const void* k, const void* v,
                 const float* lr, const float* beta,
                 const float* w1, const float* w2, const float* w3,
                 void* out, float* w1_out, float* w2_out, float* w3_out,
                 void* workspace, size_t workspace_bytes, void* stream);

/* Context parallelism ([P2 §2.2.2]: each device takes the gradient of its
 * shard of the chunk, the gradients are summed across devices, then the
 * update is applied; [P3] 「视频实验和分布式计算」).  G ranks each hold one equal share of every chunk's
 * tokens and call lact_ttt_fwd_ex with their local q, k, v, lr, beta (local
 * T = T / G, local chunk = chunk / G) and the same initial state.  The
 * library calls the hook, on the calling thread while it enqueues the work,
 * with a device buffer of `count` floats whose contents are produced by the
 * work already enqueued on `stream`:
 *   - after each chunk's gradient, on its partial gradient planes, op SUM
 *     (the summed gradient is then the whole chunk's);
 *   - once before the chunk loop (momentum rule), on the per-chunk sums of
 *     beta and their token counts [2, B*H, nchunks], op SUM (the library
 *     then divides each sum by its count on the device: the mean of beta
 *     over the whole chunk).
 * The hook must reduce the buffer in place over the ranks so that work
 * enqueued on `stream` after it returns sees the result (for example NCCL on
 * that stream), and return 0; any other value stops the call with
 * LACT_ECOMM.  Every rank then applies the same rule to the same reduced
 * gradient, so all ranks hold the same fast weights; each rank's `out` holds
 * its own queries.  Every rank must make the same sequence of calls with
 * the same problem shape and options (the hook is called the same number of
 * times with the same counts on every rank). */
/* Reduction ops a hook may be asked for.  The library asks for SUM only;
 * MEAN is kept so that hooks written against it keep their meaning. */
enum { LACT_REDUCE_SUM = 0, LACT_REDUCE_MEAN = 1 };
typedef int (*lact_allreduce_fn)(float* data, int64_t count, int op, void* stream, void* user);

/* Options of lact_ttt_fwd_ex.  Zero-initialise the struct and set what is
 * used; a NULL field leaves its feature off, and a NULL options pointer is
 * lact_ttt_fwd.
 *
 * update_mask  HOST array of ceil(T / chunk) bytes, one per chunk, shared by
 *              every (b, h).  A chunk whose byte is 0 is applied in its
 *              place in the order but skips the whole update (gradient,
 *              rule, momentum, renorm), so the state passes through it
 *              unchanged: in autoregressive video only the clean-frame
 *              chunks write the memory and the noisy ones read it
 *              ([P3] 「更新顺序必须遵守信息可见范围」; [P1 §3.2]).  Read
 *              during the call only (the launches are planned from it).
 * out_scale    DEVICE [B, H, Tq] float32, 4-byte aligned: the per-head,
 *              per-token output factor of [P1 §2.1] (the values after the
 *              page's silu of a linear map of x).  out[b,h,t,:] =
 *              out_scale[b,h,t] * f_W(q_t), the product formed in fp32 before
 *              the output's one rounding.  It may not overlap any output.
 * m1, m2, m3   DEVICE momentum state, in place, rule LACT_RULE_MOMENTUM only,
 *              all three or none: m1, m3 [B*H, dh, d], m2 [B*H, d, dh]
 *              float32, 16-byte aligned, the layouts of w*_out.  Read as the
 *              momentum before the first chunk (instead of zeros) and
 *              overwritten with the momentum after the last chunk, so a
 *              sequence split at chunk boundaries into several calls (w*_out
 *              and m* handed from one call to the next) gives the results of
 *              one call.  They may not overlap each other or any other
 *              argument.
 * allreduce    context-parallel hook (see lact_allreduce_fn above), called
 *              with `allreduce_user` as its last argument; NULL: one rank. */
typedef struct lact_fwd_opts {
  const uint8_t* update_mask;
  const float* out_scale;
  float* m1;
  float* m2;
  float* m3;
  lact_allreduce_fn allreduce;
  void* allreduce_user;
} lact_fwd_opts;

/* lact_ttt_fwd with options (see lact_fwd_opts); the same arguments,
 * layouts, workspace and error behaviour otherwise.  LACT_EINVAL also for:
 * momentum buffers with another rule, only some of m1/m2/m3, misaligned or
 * overlapping option buffers. */
int lact_ttt_fwd_ex(const lact_problem* p, const lact_fwd_opts* opts,
                    const void* q, const void* k, const void* v,
                    const float* lr, const float* beta,
                    const float* w1, const float* w2, const float* w3,
                    void* out, float* w1_out, float* w2_out, float* w3_out,
                    void* workspace, size_t workspace_bytes, void* stream);

/* Size of the library's built-in device scratch buffer used by
 * lact_ttt_fwd_noalloc (32 MiB). */
#define LACT_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20)

/* The same forward as lact_ttt_fwd for callers that cannot allocate device
 * memory.  The pages describe no such entry point; it exists for code that
 * must not call the CUDA allocator: cudaMalloc/cudaFree synchronise the
 * whole device, so latency-bound loops (a serving engine's decode step)
 * avoid them, and a plugin inside a host framework that owns the device
 * memory budget may be given no allocator at all.
 *
 * Instead of a caller workspace it uses one library-owned, file-scope
 * device buffer of LACT_NOALLOC_SCRATCH_BYTES bytes, which every GPU that
 * loads the library holds until the process exits.  Inputs and outputs are
 * still the caller's device buffers (same layouts as lact_ttt_fwd).  Returns
 * LACT_ETOOBIG, before enqueuing anything, when lact_ttt_workspace_bytes(p)
 * exceeds the buffer.  It calls no cudaMalloc, cudaFree or other allocating
 * routine.
 *
 * Every call looks up the buffer's device address on the current device
 * (cudaGetSymbolAddress, which allocates nothing); the first call on a
 * device may load the library's device code there, so make it before any
 * stream capture.  All calls share the one buffer and it keeps
 * the previous call's contents (the forward never relies on its contents at
 * entry): calls that can overlap on the GPU (different streams, or several
 * host threads) race on it and must be serialised by the caller. */
int lact_ttt_fwd_noalloc(const lact_problem* p,
                         const void* q, const void* k, const void* v,
                         const float* lr, const float* beta,
                         const float* w1, const float* w2, const float* w3,
                         void* out, float* w1_out, float* w2_out, float* w3_out,
                         void* stream);

/* Device scratch bytes lact_ttt_fwd_host needs: lact_ttt_workspace_bytes(p)
 * plus room for device copies of every input and output. */
size_t lact_ttt_host_workspace_bytes(const lact_problem* p);

/* The same forward with every tensor pointer a HOST pointer (pinned memory
 * gives full-speed copies).  Copies the inputs into `workspace` (device
 * memory of lact_ttt_host_workspace_bytes(p) bytes), runs lact_ttt_fwd on
 * `stream`, copies out and w*_out back to the host, and returns after the
 * stream has reached that point (the host buffers are then valid). */
int lact_ttt_fwd_host(const lact_problem* p,
                      const void* q, const void* k, const void* v,
                      const float* lr, const float* beta,
                      const float* w1, const float* w2, const float* w3,
                      void* out, float* w1_out, float* w2_out, float* w3_out,
                      void* workspace, size_t workspace_bytes, void* stream);

/* Device scratch bytes lact_ttt_bwd needs for problem *p (0 if *p is
 * invalid).  Pure host arithmetic. */
size_t lact_ttt_bwd_workspace_bytes(const lact_problem* p);

/* The layer's backward: the gradients of a scalar loss L with respect to
 * every input, given dL/d out (`dout`) and, optionally, dL/d w*_out
 * (`dw*_out`, all three or none).  It is the vector-Jacobian product of
 * lact_ttt_fwd_ex with the same problem, inputs and options, computed in
 * fp32: the forward's updates are recomputed (the states before each chunk
 * are kept in the workspace), then a reverse chunk loop takes, per chunk,
 * the apply's backward, the renorm and rule backward, and the backward of
 * the chunk gradient (its second-order terms: [P2 §2.1] eqs. 4-5 written as
 * functions of W, k, v and lr).  Rules: GD, momentum and Muon; for Muon the
 * rule backward is the vector-Jacobian product of the Frobenius
 * normalisation and the five Newton-Schulz steps ([P2 §2.2.1] eqs. 9-10),
 * recomputed per chunk from the kept chunk gradient.  A Muon problem runs
 * its whole backward in fp32 on the CUDA cores, bf16 inputs included (read
 * as fp32): the iteration's Jacobian magnifies bf16 operand rounding past
 * the bf16 tolerance.  GD and momentum bf16 problems run their contractions
 * on the tensor cores (bf16 operands, fp32 accumulation).  Options:
 * update_mask, out_scale, m1/m2/m3, which the backward READS as the
 * momentum the forward started from (M_0; the forward overwrote its copy,
 * so the caller keeps one; their gradient comes from lact_ttt_bwd_ex), and
 * the all-reduce hook.  Context parallelism: each rank passes the inputs of
 * its forward call and the gradients of its own share of the loss (dout for
 * its queries, its part of dw*_out and dm*_out); it gets the gradients of
 * its own tokens, and the gradients of the shared initial weights and
 * momentum, the same on every rank.  The hook is called (op SUM) on each
 * updated chunk's gradient and the beta sums and counts, as in the
 * forward's recompute; then in the reverse loop before each updated
 * chunk's renorm backward and once after the loop, on the ranks' own
 * contributions to the weights' gradient [3*B*H*d*dh floats]; and once on
 * dm*_out when given.
 * Layouts: the inputs as in lact_ttt_fwd; dout [B,H,Tq,d] in the problem's
 * dtype; dw*_out in the layouts of w*_out, or NULL (zero).  Outputs, all
 * float32 device buffers: dq [B,H,Tq,d], dk, dv [B,H,T,d], dlr [B,H,T,3],
 * dbeta [B,H,T] (momentum; else may be NULL), dw1, dw3 [Hw,dh,d], dw2
 * [Hw,d,dh] (Hw as the initial weights: summed over the batch when the
 * batch shares them), dout_scale [B,H,Tq] (required when out_scale is
 * given, else ignored).  No output may overlap an input or another output.
 * `workspace` is device scratch of lact_ttt_bwd_workspace_bytes(p) bytes,
 * 256-byte aligned.  Asynchronous on `stream`, like the forward.
 * On bf16 problems some fp32 sums are accumulated with atomic adds: dlr
 * across hidden-unit slices, and the contractions whose token range is
 * split across CTAs.  Repeated calls on the same inputs can therefore
 * differ in the last bits (the order of fp32 additions varies); the fp32
 * path is deterministic. */
int lact_ttt_bwd(const lact_problem* p, const lact_fwd_opts* opts,
                 const void* q, const void* k, const void* v,
                 const float* lr, const float* beta,
                 const float* w1, const float* w2, const float* w3,
                 const void* dout, const float* dw1_out, const float* dw2_out,
                 const float* dw3_out,
                 float* dq, float* dk, float* dv, float* dlr, float* dbeta,
                 float* dw1, float* dw2, float* dw3, float* dout_scale,
                 void* workspace, size_t workspace_bytes, void* stream);

/* Momentum gradients of the backward (R15 resume, momentum rule): the
 * gradient with respect to the final momentum the forward wrote into
 * m1/m2/m3 (dm*_out: all three or none, NULL = zero), and the output, the
 * gradient with respect to the momentum it started from (dm*: all three
 * required).  Layouts: dm1, dm3 [B*H, dh, d], dm2 [B*H, d, dh] float32,
 * 16-byte aligned device buffers, like m1/m2/m3.  Carrying the momentum
 * back through a masked chunk is the identity; through an updated chunk c,
 * M_c = mean(beta over c) M_{c-1} + G_c gives dL/dM_{c-1} = mean(beta) dL/dM_c. */
typedef struct lact_bwd_momentum {
  const float* dm1_out;
  const float* dm2_out;
  const float* dm3_out;
  float* dm1;
  float* dm2;
  float* dm3;
} lact_bwd_momentum;

/* lact_ttt_bwd that also returns the momentum gradients (`mg`, or NULL for
 * lact_ttt_bwd's behaviour).  With `mg` the rule must be
 * LACT_RULE_MOMENTUM; opts->m1/m2/m3 give M_0 (zeros if absent).
 * LACT_EINVAL also for: only some of the dm* or dm*_out buffers,
 * misaligned ones, or outputs that overlap any other argument. */
int lact_ttt_bwd_ex(const lact_problem* p, const lact_fwd_opts* opts, const lact_bwd_momentum* mg,
                    const void* q, const void* k, const void* v,
                    const float* lr, const float* beta,
                    const float* w1, const float* w2, const float* w3,
                    const void* dout, const float* dw1_out, const float* dw2_out,
                    const float* dw3_out,
                    float* dq, float* dk, float* dv, float* dlr, float* dbeta,
                    float* dw1, float* dw2, float* dw3, float* dout_scale,
                    void* workspace, size_t workspace_bytes, void* stream);

/* Sliding-window attention, the other half of the LaCT block ([P1 §1.1]):
 * per head and channel learnable scales and offsets on the queries and
 * keys, q' = q * q_scale + q_offset, k' = k * k_scale + k_offset, then for
 * every token t, out_t = sum_j softmax_j(q'_t . k'_j / sqrt(d)) v_j over the
 * `window` most recent tokens, t - window < j <= t (causal; the window
 * includes the token itself).  q, k, v, out [B, H, T, d] bf16 (device);
 * q_scale, q_offset, k_scale, k_offset [H, d] float32 (device).  Limits: d
 * a multiple of 64 up to 512, T and window multiples of 128, window <=
 * 16384, B*H <= 4096.  For d <= 256 the scores stay on chip and the
 * workspace holds one transformed copy of q (B*H*T*d bf16); for d = 320..512
 * the scores take a round trip through it (fp32 scores, bf16
 * probabilities: B*H*T*(window+128)*6 bytes, plus padded copies of k' and
 * v).  lact_swa_workspace_bytes gives its size.  Asynchronous on `stream`;
 * the error behaviour of lact_ttt_fwd. */
typedef struct lact_swa_problem {
  int64_t B, H, T, d, window;
  int32_t dtype;   /* LACT_BF16 */
  int32_t reserved;
} lact_swa_problem;

size_t lact_swa_workspace_bytes(const lact_swa_problem* p);

int lact_swa_fwd(const lact_swa_problem* p, const void* q, const void* k, const void* v,
                 const float* q_scale, const float* q_offset,
                 const float* k_scale, const float* k_offset,
                 void* out, void* workspace, size_t workspace_bytes, void* stream);

/* Waits for `stream`, then returns and clears the device status word of the
 * current device: LACT_OK, or LACT_ETIMEOUT if a bounded wait inside one of
 * this library's kernels gave up since the last call (its results are then
 * invalid), or LACT_ECUDA if the stream reported an error. */
int lact_ttt_status(void* stream);

/* LACT_OK if the current CUDA device is an sm_100 part this library was
 * built for, LACT_ENODEV otherwise (or LACT_ECUDA if there is no device). */
int lact_device_check(void);

/* Kernel launches one lact_ttt_fwd call of problem *p enqueues (0 if *p is
 * invalid).  Pure host arithmetic. */
int64_t lact_ttt_launch_count(const lact_problem* p);

/* The same for lact_ttt_fwd_ex with options *opts (NULL = none): masked
 * chunks launch no update kernels. */
int64_t lact_ttt_launch_count_ex(const lact_problem* p, const lact_fwd_opts* opts);

/* Failure-path self-test: launches one block whose thread waits on a shared
 * memory barrier that nothing ever completes, with a wait budget of
 * `budget_cycles` SM clock cycles (1 <= budget_cycles <= 2^31).  The wait
 * gives up, records LACT_ETIMEOUT in the device status word and the kernel
 * returns; the context stays usable.  Returns the launch status; read the
 * outcome with lact_ttt_status(stream).  Restores the normal budget after
 * the launch. */
int lact_selftest_wait_timeout(int64_t budget_cycles, void* stream);

/* Launch profiler.  While enabled, every kernel launch of lact_ttt_fwd is
 * bracketed by a pair of CUDA events recorded on the launching stream, and
 * all launches of a call go to the caller's stream one after another (no
 * side-stream overlap), so each pair times one kernel running alone.
 * lact_profile_read waits for those events, returns per kernel kind the
 * number of launches and the summed device milliseconds since the last read
 * (arrays of lact_kernel_kinds() entries), and forgets them.  Off by default;
 * not meant for use while a stream is being captured. */
int lact_profile_enable(int on);
int lact_profile_read(int64_t* launches, double* ms, int nkinds);
int lact_kernel_kinds(void);
const char* lact_kernel_name(int kind);

/* Static text for a status code. */
const char* lact_status_string(int code);

#ifdef __cplusplus
}
#endif

#endif /* LACT_H */
