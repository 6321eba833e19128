/*
 * moe.h -- C ABI of the B200 (sm_100a) inference MoE layer library, libmoe.so.
 *
 * The layer is the routed half of a DeepSeek-V3-style MoE block as the pages
 * show it:
 *   router   "Kimi K2 · Affinities", gate-forward excerpt (MoEGate.forward,
 *            noaux_tc) and "DeepSeek-V3.2-Exp · Affinities", gate-forward
 *            excerpt (Gate.forward): fp32 logits x.W^T, sigmoid, selection-only
 *            correction bias, group score = sum of the group's top two, top
 *            topk_group groups, top top_k experts, unbiased weights
 *            renormalised and multiplied by the route scale;
 *   dispatch "Kimi K3 · Add shared output", moe-forward excerpt (moe_infer):
 *            per-expert counts, sort of the token slots by expert, row gather;
 *   experts  "Kimi K3 · Gate features", expert excerpt (KimiBlockSparseMLP)
 *            and situ excerpt (SituAndMul): w1/w3 projections, SiLU-and-mul or
 *            SiTU, w2 projection;
 *   combine  moe_infer again: unpermute, fp32 weighted sum over k, cast.
 *
 * Conventions shared by every entry point
 *   - Tensor pointers are DEVICE pointers owned by the caller; the library
 *     never allocates, frees or keeps them.  Row-major, densely packed.
 *     bf16 tensors are passed as uint16_t bit patterns (moe_bf16).
 *   - Scratch memory is passed in as (ws, ws_bytes), a device buffer of at
 *     least the size the matching *_workspace_size function returns, 256-byte
 *     aligned.  Its first 256 bytes hold the device status word.
 *   - Every call enqueues its kernels on `stream` (a cudaStream_t, NULL = the
 *     legacy default stream) and returns without synchronising.  No entry point
 *     copies data to the host or waits for the GPU, so a sequence of calls can
 *     be captured in a CUDA graph.
 *   - Return value: MOE_OK or a negative moe_status.  Argument errors are found
 *     on the host before anything is enqueued.  Errors found by the kernels
 *     themselves (an expert index out of range, inconsistent offsets, a wait
 *     that ran out) are recorded in the status word of the workspace; they are
 *     sticky until moe_get_status() reads and clears them.
 *   - N = 0 (no tokens) is a valid, empty call.
 *   - Index tensors are int32 (the pages use int64).
 *   - Stateless and thread-safe; device attributes are read once per device.
 */
#ifndef MOE_H
#define MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

typedef uint16_t moe_bf16;

typedef enum moe_status {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = -1,    /* null pointer, negative size, inconsistent config */
  MOE_ERR_UNSUPPORTED = -2,    /* shape outside the kernels' limits (see below)   */
  MOE_ERR_ALIGNMENT = -3,      /* pointer not 16-byte aligned                      */
  MOE_ERR_WORKSPACE = -4,      /* ws too small or not 256-byte aligned             */
  MOE_ERR_CUDA = -5,           /* a CUDA call or launch failed                     */
  MOE_ERR_DEVICE_TIMEOUT = -6, /* a kernel's bounded wait ran out (status word)    */
  MOE_ERR_DEVICE_BOUNDS = -7,  /* a kernel met an index out of range (status word) */
  MOE_ERR_NO_DEVICE = -8       /* no sm_100 device is current                      */
} moe_status;

/* Routing configuration ("Kimi K2 · Affinities", gate-init excerpt: the
 * MoEGate fields; "DeepSeek-V3.2-Exp · Affinities", gate-init excerpt).
 * Limits: 1 <= num_experts <= 1024; num_experts % n_group == 0;
 * 1 <= n_group <= 32; if n_group > 1 each group holds >= 2 experts;
 * 1 <= topk_group <= n_group; 1 <= top_k <= 16;
 * top_k <= topk_group * num_experts / n_group. */
typedef struct moe_route_cfg {
  int num_experts;     /* E: n_routed_experts                                  */
  int n_group;         /* G: groups of E/G consecutive experts                 */
  int topk_group;      /* TG: groups kept per token                            */
  int top_k;           /* K: experts per token (num_experts_per_tok)           */
  int norm_topk_prob;  /* nonzero: renormalise the K weights when K > 1        */
  float route_scale;   /* routed_scaling_factor / route_scale                  */
  int score_func;      /* MOE_SCORE_SIGMOID (0, default) or MOE_SCORE_SOFTMAX   */
  int group_score;     /* MOE_GROUP_TOP2_SUM (0, default) or MOE_GROUP_MAX      */
} moe_route_cfg;

/* Scoring variants ("DeepSeek-V3.2-Exp · Affinities", gate-forward):
 *   MOE_SCORE_SOFTMAX: s = softmax over all E logits (fp32 rounding of
 *     exp(L_e - max) / sum_j exp(L_j - max), evaluated in double with the sum
 *     taken in expert order) in place of the sigmoid; that page renormalises
 *     only sigmoid scores, so softmax routing in its form sets
 *     norm_topk_prob = 0;
 *   MOE_GROUP_MAX: group score = the group's largest choice score (the page's
 *     amax, used there when the gate has no correction bias) in place of the
 *     sum of its two largest. */
enum { MOE_SCORE_SIGMOID = 0, MOE_SCORE_SOFTMAX = 1 };
enum { MOE_GROUP_TOP2_SUM = 0, MOE_GROUP_MAX = 1 };

/* Expert activation ("Kimi K3 · Gate features", situ excerpt).
 * kind MOE_ACT_SILU: h = bf16(bf16(silu(g)) * u), silu(g) = g * sigmoid(g).
 * kind MOE_ACT_SITU: h = bf16(beta*tanh(g/beta)*sigmoid(g) * u'),
 *   u' = linear_beta*tanh(u/linear_beta) when linear_beta is set, else u;
 *   evaluated in fp32.  beta == 0 or NaN means 1.0 (the page's "beta or 1.0");
 *   linear_beta == 0 or NaN means "not set". */
typedef enum moe_act_kind { MOE_ACT_SILU = 0, MOE_ACT_SITU = 1 } moe_act_kind;
typedef struct moe_act_cfg {
  int kind;
  float beta;
  float linear_beta;
} moe_act_cfg;

/* Shape limits: d (hidden width of the experts) and F (d_ff) are multiples
 * of 128; d_r (router width) is a multiple of 32; all bf16 row pointers
 * 16-byte aligned. */

/* ------------------------------------------------------------------ router */

/* Scratch bytes needed by moe_route (and by moe_route_from_logits, which
 * needs only the status word). */
MOE_API size_t moe_route_workspace_size(int64_t N, int d_r, const moe_route_cfg* cfg);

/* Router: for each of the N tokens,
 *   L = fp32(x . W^T)                      ([N, d_r] bf16 x [E, d_r] fp32)
 *   s = sigmoid(L) (fp32), c = s + bias    (bias only steers the choice)
 *   if n_group > 1: group score = sum of the two largest c of the group; the
 *     topk_group best groups are kept, the other experts get c = -inf
 *   topk_idx = the top_k largest c, ordered by (c descending, index ascending)
 *     -- ties go to the lowest expert index
 *   topk_w[k] = s[topk_idx[k]]; if top_k > 1 and norm_topk_prob:
 *     topk_w /= (sum_k topk_w + 1e-20), summed in k order; topk_w *= route_scale
 * x: [N, d_r] bf16; W: [E, d_r] fp32; bias: [E] fp32 or NULL;
 * topk_idx: [N, K] int32 out; topk_w: [N, K] fp32 out.
 * The logits are fp32-accurate (the page's fp32 F.linear; see moe_gate_logits). */
MOE_API int moe_route(const moe_bf16* x, int64_t N, int d_r, const float* W, const float* bias,
                      const moe_route_cfg* cfg, int32_t* topk_idx, float* topk_w, void* ws,
                      size_t ws_bytes, void* stream);

/* The router's gate GEMM alone ("Kimi K2 · Affinities", gate-forward: the
 * F.linear of the fp32-upcast hidden states with the fp32 weight):
 * logits[t, e] = fp32(sum_j x[t, j] * W[e, j]), x: [N, d_r] bf16, W: [E, d_r]
 * fp32, logits: [N, E] fp32 out.  Same kernels as moe_route: fp32 FMA chains
 * of 32 terms added in double for small batches; for batches that fill the
 * GPU, exact int8 tensor-core products of 7-bit digits of x and W (error
 * below ~2e-8 for unit-scale logits).  Scratch: moe_gate_logits_workspace_size. */
MOE_API size_t moe_gate_logits_workspace_size(int64_t N, int d_r, int E);
MOE_API int moe_gate_logits(const moe_bf16* x, int64_t N, int d_r, const float* W, int E,
                            float* logits, void* ws, size_t ws_bytes, void* stream);

/* Selection and weights only, from caller-supplied fp32 logits [N, E]: the
 * same computation as moe_route after its gate GEMM.  Bit-exact: sigmoid is
 * the fp32 rounding of 1/(1+exp(-L)) evaluated in double. */
MOE_API int moe_route_from_logits(const float* logits, int64_t N, const float* bias,
                                  const moe_route_cfg* cfg, int32_t* topk_idx, float* topk_w,
                                  void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------- dispatch */

MOE_API size_t moe_dispatch_workspace_size(int64_t N, int K, int E);

/* moe_infer's dispatch with no host round trip:
 *   counts[e]  = number of slots (t,k) with topk_idx[t,k] == e
 *   offsets    = exclusive prefix sum of counts, offsets[E] = S = N*K
 *   perm[j]    = slot t*K+k at sorted position j; the sort is STABLE: slots of
 *                one expert keep ascending slot order
 *   pos[slot]  = its sorted position (pos[perm[j]] == j)
 *   xs[j, :]   = x_e[perm[j] / K, :]
 * topk_idx: [N, K] int32; x_e: [N, d_e] bf16; counts [E], offsets [E+1],
 * perm [S], pos [S] int32 out; xs [S, d_e] bf16 out.
 * xs may be NULL: then only counts, offsets, perm and pos are written and
 * x_e is not read (it may be NULL too), for callers that move the rows
 * themselves (moe_expert_ffn_gathered, moe_ep_dispatch_rows).
 * An expert index outside [0, E) is recorded as MOE_ERR_DEVICE_BOUNDS and its
 * slot is left out of every output. */
MOE_API int moe_dispatch(const int32_t* topk_idx, int64_t N, int K, int E, const moe_bf16* x_e,
                         int d_e, int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* pos,
                         moe_bf16* xs, void* ws, size_t ws_bytes, void* stream);

/* Fixed size of the device array that moe_dispatch_static uses as scratch. */
#define MOE_DISPATCH_STATIC_SCRATCH_BYTES (2u << 20)

/* moe_dispatch for callers that cannot allocate device memory.
 * The pages have no counterpart: this entry point exists for library users
 * who have no way to provide the workspace that moe_dispatch takes, e.g. a
 * plugin that its host framework hands only input and output tensors, a
 * serving process whose device memory is fully reserved by another
 * allocator, or a latency-critical loop that must not call cudaMalloc (it can
 * synchronise the device).
 * Arguments, outputs and results are those of moe_dispatch without (ws,
 * ws_bytes); it enqueues the same kernels and allocates nothing (no
 * cudaMalloc, cudaFree or allocating library routine).
 * Scratch: a file-scope device array of MOE_DISPATCH_STATIC_SCRATCH_BYTES
 * (2 MiB) inside libmoe.so, held by every GPU that loads the library until
 * the process exits.  Calls whose per-chunk counts (4 * chunks * E bytes,
 * chunks = ceil(N*K / clamp(N*K/256, 64, 1024) rounded up to 32)) exceed it
 * return MOE_ERR_UNSUPPORTED; 131072 slots over 384 experts use 0.4 MiB.
 * Set-up: the first call made with a given CUDA context current (normally
 * the device's primary context) looks up the array's device address in that
 * context (cudaGetSymbolAddress) and caches it for that context; make that
 * first call before any stream capture.  A lookup that fails is not cached:
 * the call returns MOE_ERR_CUDA, leaves no pending CUDA error, and a later
 * call tries again.
 * xs may be NULL exactly as in moe_dispatch: then only counts, offsets, perm
 * and pos are written and x_e is not read.
 * Every call shares the one array and overwrites it, so calls that can
 * overlap on the GPU (different streams, or different host threads without
 * ordering) race and corrupt each other's results; serialise them on one
 * stream.  An expert index outside [0, E) is skipped as in moe_dispatch but
 * is not reported (there is no status word). */
MOE_API int moe_dispatch_static(const int32_t* topk_idx, int64_t N, int K, int E,
                                const moe_bf16* x_e, int d_e, int32_t* counts, int32_t* offsets,
                                int32_t* perm, int32_t* pos, moe_bf16* xs, void* stream);

/* ------------------------------------------------------------- expert MLP */

MOE_API size_t moe_expert_ffn_workspace_size(int64_t S, int d_e, int E, int F);

/* Grouped expert MLP over the sorted rows: for every expert e, the rows
 * offsets[e] .. offsets[e+1]-1 of xs go through
 *   g = bf16(xs . w1[e]^T), u = bf16(xs . w3[e]^T)   (fp32 accumulation)
 *   h = act(g, u) (see moe_act_cfg), y = bf16(h . w2[e]^T)
 * xs: [S, d_e] bf16; offsets: [E+1] int32 (non-decreasing, offsets[0] = 0,
 * offsets[E] = S); w1, w3: [E, F, d_e] bf16; w2: [E, d_e, F] bf16;
 * y: [S, d_e] bf16 out.  Experts with no rows cost nothing. */
MOE_API int moe_expert_ffn(const moe_bf16* xs, const int32_t* offsets, int E, int64_t S, int d_e,
                           int F, const moe_bf16* w1, const moe_bf16* w3, const moe_bf16* w2,
                           const moe_act_cfg* act, moe_bf16* y, void* ws, size_t ws_bytes,
                           void* stream);

/* ----------------------------------------------------------------- combine */

MOE_API size_t moe_combine_workspace_size(void);

/* Unpermute and combine:
 *   out[t, :] = bf16( sum_{k=0..K-1} fp32(y[pos[t*K+k], :]) * topk_w[t, k] )
 * with every product rounded to fp32 and the sum taken in k order in fp32.
 * y: [S, d_e] bf16; pos: [S] int32; topk_w: [N, K] fp32; out: [N, d_e] bf16.
 * pos == NULL: y is already in slot order (the page's new_x, as
 * moe_expert_ffn_to_slots writes it), so row t*K+k is read for slot (t, k). */
MOE_API int moe_combine(const moe_bf16* y, const int32_t* pos, const float* topk_w, int64_t N,
                        int K, int d_e, moe_bf16* out, void* ws, size_t ws_bytes, void* stream);

/* moe_expert_ffn with the scatter inside the w2 kernel ("Kimi K3 · Add shared
 * output", moe-forward excerpt: new_x[idxs] = outs): the output row of sorted
 * row j is stored at row perm[j] of y_slots, so y_slots is the MLP output in
 * slot order (token t's K rows are rows t*K .. t*K+K-1) and moe_combine reads
 * it with pos == NULL.  perm: [S] int32 as moe_dispatch writes it (a
 * permutation of 0 .. S-1; an entry outside it is recorded as
 * MOE_ERR_DEVICE_BOUNDS and its row is not stored).  y_slots: [S, d_e] bf16.
 * Arithmetic, arguments and workspace otherwise as moe_expert_ffn. */
MOE_API int moe_expert_ffn_to_slots(const moe_bf16* xs, const int32_t* offsets,
                                    const int32_t* perm, int E, int64_t S, int d_e, int F,
                                    const moe_bf16* w1, const moe_bf16* w3, const moe_bf16* w2,
                                    const moe_act_cfg* act, moe_bf16* y_slots, void* ws,
                                    size_t ws_bytes, void* stream);

/* moe_expert_ffn with the gather inside the w1/w3 kernel: row j of segment
 * e is x_e[perm[j] / K] (perm and offsets as moe_dispatch writes them), read
 * by tile::gather4 TMA loads, so no S x d_e copy of the tokens is made.
 * x_e [N, d_e] bf16.  Decode and mid-size batches only (S <= 128 * E, else
 * MOE_ERR_UNSUPPORTED).  It saves the copy's memory, not time: on a B200 the
 * separate token-major gather plus tiled loads is faster (the layer,
 * moe_forward, uses that).  Workspace as moe_expert_ffn. */
MOE_API int moe_expert_ffn_gathered(const moe_bf16* x_e, int64_t N, int K, const int32_t* perm,
                                    const int32_t* offsets, int E, int d_e, int F,
                                    const moe_bf16* w1, const moe_bf16* w3, const moe_bf16* w2,
                                    const moe_act_cfg* act, moe_bf16* y, void* ws,
                                    size_t ws_bytes, void* stream);

/* ------------------------------------------- expert parallelism, receive side
 *
 * With the experts split over P ranks (rank q holds experts q*E_local ..
 * q*E_local + E_local - 1, "Kimi K3 · Add shared output", moe-forward excerpt:
 * self.experts[i + self.ep_rank * self.experts_per_rank]), a rank's rows
 * sorted by moe_dispatch are already grouped by destination rank, so one
 * all-to-all sends each rank its slice; the rows a rank receives arrive
 * grouped by source rank and, within a source, sorted by local expert.
 * moe_ep_expert_ffn runs the local experts' MLP on them in that order:
 *   xr [R, d_e] bf16       the received rows, R = sum of recv_counts;
 *   recv_counts [P, E_local] int32 (device): rows source p sent for local
 *                          expert e, the segment (p, e) of xr;
 *   w1, w3 [E_local, F, d_e], w2 [E_local, d_e, F]: this rank's experts;
 *   y [R, d_e] bf16        the outputs, in xr's order (to be sent back).
 * P * E_local <= 1024.  Counts that do not add up to R are reported in the
 * status word (MOE_ERR_DEVICE_BOUNDS) and no row is read out of range.
 * Workspace: moe_ep_expert_ffn_workspace_size(R, d_e, P, E_local, F). */
MOE_API size_t moe_ep_expert_ffn_workspace_size(int64_t R, int d_e, int P, int E_local, int F);
MOE_API int moe_ep_expert_ffn(const moe_bf16* xr, int64_t R, const int32_t* recv_counts, int P,
                              int E_local, int d_e, int F, const moe_bf16* w1,
                              const moe_bf16* w3, const moe_bf16* w2, const moe_act_cfg* act,
                              moe_bf16* y, void* ws, size_t ws_bytes, void* stream);

/* ----------------------------------------- expert parallelism over peer memory
 *
 * The same exchange without a collective library: the sending rank's kernel
 * stores each token row straight into the receiving rank's row buffer, and
 * the combine loads the expert outputs straight from the rank that computed
 * them, through device addresses of the peers' buffers (NVLink peer mappings
 * on a multi-GPU node; any device addresses the GPU can reach).
 *
 * Rank q holds experts q*E_local .. q*E_local + E_local - 1, E_local = E / P.
 * On the sending rank, sorted position j (0 <= j < S, moe_dispatch's pos and
 * offsets) belongs to the rank q with offsets[q*E_local] <= j <
 * offsets[(q+1)*E_local], and its row in rank q's buffer is
 *   first_row[q] + j - offsets[q*E_local].
 * The caller sizes the buffers and chooses first_row so that the senders'
 * segments do not overlap; with first_row[q] = the rows that ranks 0 .. p-1
 * send to q (p this rank), rank q's buffer holds its received rows grouped by
 * source rank and sorted by local expert, the layout moe_ep_expert_ffn takes.
 * Ordering between ranks (all rows stored before a rank's experts read them,
 * all outputs written before the senders' combines load them) is the
 * caller's: a barrier across the ranks between the steps.
 * Host checks of both calls: MOE_ERR_INVALID_ARG for E % P != 0, a negative
 * first_row or capacity, a NULL buffer with capacity > 0 or a NULL tensor
 * pointer; MOE_ERR_UNSUPPORTED for P outside 1 .. MOE_MAX_PEERS, K > 16,
 * E > 1024 or d_e % 8 != 0; MOE_ERR_ALIGNMENT for a buffer, x_e or out not
 * 16-byte aligned; MOE_ERR_WORKSPACE for a missing or short workspace.
 * N = 0 is a successful no-op. */
#define MOE_MAX_PEERS 64

typedef struct moe_peer_rows {
  int num_ranks;                    /* P, 1 .. MOE_MAX_PEERS; E % P == 0           */
  void* rows[MOE_MAX_PEERS];        /* rank q's [capacity[q], d_e] bf16 buffer, as  */
                                    /* a device address of this GPU (16-B aligned)  */
  int64_t first_row[MOE_MAX_PEERS]; /* this rank's first row in rank q's buffer     */
  int64_t capacity[MOE_MAX_PEERS];  /* rows in rank q's buffer                      */
} moe_peer_rows;

/* Send side: for every slot s = t*K + k with pos[s] = j >= 0, rank q's row
 * first_row[q] + j - offsets[q*E_local] becomes x_e[t, :] (each token row is
 * read from HBM once and stored K times).  x_e [N, d_e] bf16; pos [S],
 * offsets [E+1] int32 as moe_dispatch writes them.  A row outside
 * [0, capacity[q]) is not stored and is recorded as MOE_ERR_DEVICE_BOUNDS.
 * Workspace: moe_combine_workspace_size() bytes (the status word). */
MOE_API int moe_ep_dispatch_rows(const moe_bf16* x_e, int64_t N, int K, int d_e,
                                 const int32_t* pos, const int32_t* offsets, int E,
                                 const moe_peer_rows* peers, void* ws, size_t ws_bytes,
                                 void* stream);

/* Return side, fused with the combine: moe_combine where the row of slot s is
 * loaded from rank q's buffer at first_row[q] + pos[s] - offsets[q*E_local]
 * (peers->rows now name the buffers of expert outputs, laid out as the rows
 * were sent).  Same arithmetic as moe_combine: products rounded to fp32,
 * summed in k order, one rounding to bf16.  out [N, d_e] bf16; topk_w [N, K]
 * fp32.  Rows out of range are skipped and recorded as
 * MOE_ERR_DEVICE_BOUNDS.  Workspace: moe_combine_workspace_size() bytes. */
MOE_API int moe_ep_combine_rows(const moe_peer_rows* peers, const int32_t* pos,
                                const int32_t* offsets, int E, const float* topk_w, int64_t N,
                                int K, int d_e, moe_bf16* out, void* ws, size_t ws_bytes,
                                void* stream);

/* ------------------------------------------------------------ whole layer */

MOE_API size_t moe_workspace_size(int64_t N, int d_r, int d_e, const moe_route_cfg* cfg, int F);

/* Optional CUDA events recorded between the stages of moe_forward (each entry
 * a cudaEvent_t or NULL): after routing, after dispatch, after the w1/w3
 * kernel, after the w2 kernel, after the combine. */
typedef struct moe_stage_events {
  void* after_route;
  void* after_dispatch;
  void* after_gate_up;
  void* after_down;
  void* after_combine;
} moe_stage_events;

/* The routed MoE layer, moe_route -> moe_dispatch -> moe_expert_ffn ->
 * moe_combine, on one stream with no host synchronisation.
 * x_r: [N, d_r] bf16, the router's input.  x_e: [N, d_e] bf16, the experts'
 * input, or NULL to use x_r (then d_e must equal d_r); a latent MoE routes on
 * the full width and runs its experts on a narrower input.
 * topk_idx_out [N, K] int32 and topk_w_out [N, K] fp32 may be NULL.
 * events may be NULL. */
MOE_API int moe_forward(const moe_bf16* x_r, const moe_bf16* x_e, int64_t N, int d_r, int d_e,
                        const float* W, const float* bias, const moe_route_cfg* cfg,
                        const moe_bf16* w1, const moe_bf16* w3, const moe_bf16* w2, int F,
                        const moe_act_cfg* act, moe_bf16* out, int32_t* topk_idx_out,
                        float* topk_w_out, void* ws, size_t ws_bytes, void* stream,
                        const moe_stage_events* events);

/* ------------------------------------------------ the block around the layer
 *
 * KimiSparseMoeBlock.forward ("Kimi K3 · Add shared output", moe-forward
 * excerpt): the gate scores the full-width input x; a latent block projects x
 * down (routed_expert_down_proj) before moe_infer, then normalises
 * (routed_expert_norm) and projects up (routed_expert_up_proj); the shared
 * experts' output on x is added last.  Readings where the pages are silent:
 * both projections are bias-free Linear layers; routed_expert_norm is an
 * RMSNorm with a bf16 weight (moe_rms_norm); the shared experts are one gated
 * MLP of the routed experts' kind and activation on the full width, of hidden
 * width F_shared (the sum over shared experts). */

/* Bias-free bf16 Linear, y[m, n] = bf16( sum_k x[m, k] * W[n, k] ) with fp32
 * tensor-core accumulation, and with a residual y = bf16( bf16(sum) +
 * residual[m, n] ).  x [M, K], W [N_out, K] (nn.Linear layout), residual and
 * y [M, N_out]: bf16, row-major, device memory, 16-byte aligned.  K and N_out
 * multiples of 128.  y may be the residual buffer; it must not overlap x or
 * W.  Workspace: moe_linear_workspace_size(M, K, N_out) bytes (it holds the
 * split-K partial sums of small M; 0 for invalid shapes). */
MOE_API size_t moe_linear_workspace_size(int64_t M, int K, int N_out);
MOE_API int moe_linear(const moe_bf16* x, int64_t M, int K, const moe_bf16* W, int N_out,
                       const moe_bf16* residual, moe_bf16* y, void* ws, size_t ws_bytes,
                       void* stream);

/* The shared experts alone: one gated MLP (the routed experts' kind) on every
 * row, y = bf16( h . w2^T ) with h = act(bf16(x . w1^T), bf16(x . w3^T)), and
 * with a residual y = bf16( bf16(...) + residual ).  x and residual/y
 * [M, d], w1 and w3 [F, d], w2 [d, F], bf16; d and F multiples of 128.
 * Workspace: moe_shared_experts_workspace_size(M, d, F) bytes. */
MOE_API size_t moe_shared_experts_workspace_size(int64_t M, int d, int F);
MOE_API int moe_shared_experts(const moe_bf16* x, int64_t M, int d, int F, const moe_bf16* w1,
                               const moe_bf16* w3, const moe_bf16* w2, const moe_act_cfg* act,
                               const moe_bf16* residual, moe_bf16* y, void* ws,
                               size_t ws_bytes, void* stream);

/* RMSNorm of each row of x [N, d] (the reading of routed_expert_norm):
 *   r = 1 / sqrt(mean(x^2) + eps)   (double)
 *   out = bf16( weight * bf16(x * r) )
 * weight [d] bf16; d a multiple of 8, at most 8192; eps finite and >= 0.
 * out may equal x.  No workspace, no device-side failure. */
MOE_API int moe_rms_norm(const moe_bf16* x, int64_t N, int d, const moe_bf16* weight, float eps,
                         moe_bf16* out, void* stream);

typedef struct moe_block_dims {
  int d_r;          /* hidden size (router input, block output)              */
  int d_e;          /* routed experts' width: d_r, or the latent width        */
  int F;            /* routed experts' hidden width (moe_intermediate_size)   */
  int F_shared;     /* shared experts' hidden width, 0 = no shared experts    */
  float norm_eps;   /* routed_expert_norm epsilon                             */
} moe_block_dims;

/* Device pointers, 16-byte aligned.  NULL marks an absent part. */
typedef struct moe_block_weights {
  const float* gate_weight;     /* [E, d_r] fp32                                  */
  const float* gate_bias;       /* [E] fp32 correction bias, or NULL              */
  const moe_bf16* down_proj;    /* [d_e, d_r]; NULL: not latent (d_e == d_r)      */
  const moe_bf16* norm_weight;  /* [d_e]; NULL: no routed_expert_norm (latent only)*/
  const moe_bf16* up_proj;      /* [d_r, d_e]; given exactly when down_proj is    */
  const moe_bf16* w1;           /* routed experts [E, F, d_e]                     */
  const moe_bf16* w3;           /* [E, F, d_e]                                    */
  const moe_bf16* w2;           /* [E, d_e, F]                                    */
  const moe_bf16* shared_w1;    /* [F_shared, d_r], or NULL with the two below    */
  const moe_bf16* shared_w3;    /* [F_shared, d_r]                                */
  const moe_bf16* shared_w2;    /* [d_r, F_shared]                                */
} moe_block_weights;

/* Workspace bytes for moe_block_forward (0 if the arguments are invalid). */
MOE_API size_t moe_block_workspace_size(int64_t N, const moe_block_dims* dims,
                                        const moe_block_weights* weights,
                                        const moe_route_cfg* cfg);

/* out [N, d_r] bf16 = the block on x [N, d_r] bf16, on one stream with no host
 * synchronisation: route -> shared experts -> down_proj -> dispatch -> expert
 * MLP -> combine (+ RMSNorm) -> up_proj (+ shared output); without a latent
 * projection the combine adds the shared output.  d_r, d_e, F, F_shared
 * multiples of 128; d_e <= 8192; the routed layer's limits apply.
 * topk_idx_out / topk_w_out as in moe_forward.  act applies to the routed and
 * the shared experts. */
MOE_API int moe_block_forward(const moe_bf16* x, int64_t N, const moe_block_dims* dims,
                              const moe_block_weights* weights, const moe_route_cfg* cfg,
                              const moe_act_cfg* act, moe_bf16* out, int32_t* topk_idx_out,
                              float* topk_w_out, void* ws, size_t ws_bytes, void* stream);

/* --------------------------------------------------------------- status */

/* Reads (synchronising `stream`) and clears the device status word of a
 * workspace.  Returns MOE_OK or the first device-side error recorded. */
MOE_API int moe_get_status(void* ws, void* stream);

/* Text for a moe_status code. */
MOE_API const char* moe_strerror(int code);

/* Kernels this library has launched in this process so far, over all devices
 * and host threads (the launches the CUDA runtime accepted).  A caller that
 * accounts for GPU work reads it before and after a region: the difference is
 * the number of libmoe kernels that region enqueued.  Not part of the pages'
 * method: bookkeeping for measurement. */
MOE_API uint64_t moe_launch_count(void);

/* Diagnostics hook for the kernels' bounded waits (not part of the pages'
 * method).  Every mbarrier wait in the tensor-core kernels gives up after a
 * time limit, records MOE_ERR_DEVICE_TIMEOUT in the status word and stops the
 * kernel cleanly (its other roles stop, its tensor memory is freed), so a
 * broken protocol cannot hang the GPU.  With on != 0 the grouped expert GEMM
 * kernels launched afterwards (moe_expert_ffn, moe_forward and every entry
 * point built on them) make that path run: before issuing any copy, each
 * CTA's producer waits on a barrier that nothing arrives on, with a 1 ms
 * limit; the wait runs out, the call's status word reads
 * MOE_ERR_DEVICE_TIMEOUT and its outputs are left unwritten.  on = 0 (the
 * default) restores normal operation; the CUDA context stays usable.
 * Process-wide and read at launch: not for use while other threads launch
 * libmoe kernels.  Returns the previous setting. */
MOE_API int moe_set_wait_probe(int on);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H */
