/*
 * moe_b200.h — C ABI of the sparse Mixture-of-Experts layer forward for
 * NVIDIA B200 (sm_100a).
 *
 * The layer (page "Switch Transformers: Scaling to Trillion Parameter Models
 * with Simple and Efficient Sparsity", study notes, sec. 2.1-2.2):
 *   router      h(x) = W_r x                                  (sec. 2.1)
 *   gate        p_i(x) = exp(h_i) / sum_j exp(h_j)            (sec. 2.1, eq. 1)
 *   top-k set   T = indices of the k largest gates            (sec. 2.1; k = 1
 *               Switch, k = 2 X-MoE per "[Paper review] TorchScale",
 *               proposed method)
 *   capacity    C = (tokens / experts) x capacity_factor      (sec. 2.2, eq. 3)
 *               overflowing tokens are dropped: the layer adds 0 for them
 *   experts     E_i(x) = ReLU(x W1_i^T) W2_i^T
 *   combine     y = sum_{i in T} p_i(x) E_i(x)                (sec. 2.1, eq. 2)
 * plus Random Routed Experts ("[Paper review] PanGu-Sigma", proposed method)
 * and the SparseClip norm ("[Paper review] TorchScale", proposed method).
 *
 * Conventions for every entry point:
 *   * All tensor pointers are DEVICE pointers owned by the caller; the
 *     library never allocates, frees or retains device memory.  Scratch comes
 *     from a caller-provided workspace of the size the matching *_size query
 *     returns.  Host-side arrays are marked "host".
 *   * Tensors are dense, row-major (C order), 16-byte aligned.  Activations
 *     and weights are bf16 (dtype MOE_DTYPE_BF16) or fp32 (MOE_DTYPE_F32);
 *     logits and gates are always fp32; indices int32; masks uint8.
 *   * Work is enqueued asynchronously on `stream` (a cudaStream_t; 0 = the
 *     legacy default stream) and the call returns at once.
 *   * Arguments are validated on the host before anything is launched; a
 *     rejected call launches nothing and returns a negative MOE_ERR_* code.
 *     A failed launch returns MOE_ERR_CUDA; moe_last_error() describes it.
 *   * Conditions seen on the device are OR-ed into the optional `status`
 *     word (device int32, nullable; enum moe_status_bits).  The caller
 *     zeroes `status` before the call and reads it after synchronising.
 *   * Every wait inside a kernel is bounded (1 s by default, see
 *     moe_set_wait_limit_ns).  The status word is also the call's give-up
 *     signal: once one wait expires and sets MOE_STATUS_TIMEOUT, every other
 *     wait of every kernel that shares the word gives up at its next poll, so
 *     the whole call ends within about one limit.  A call that starts with
 *     the timeout bit already set therefore gives up its waits at once (its
 *     outputs are invalid, as the bit says).  Without a status word each
 *     thread block gives up on its own limit.
 */
#ifndef MOE_B200_H_
#define MOE_B200_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* moe_stream_t; /* identical to cudaStream_t */

#define MOE_ABI_VERSION 3

enum moe_error {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARGUMENT = -1, /* null pointer, bad size, bad enum value   */
  MOE_ERR_UNSUPPORTED = -2,      /* valid MoE, but outside this library's range */
  MOE_ERR_ALIGNMENT = -3,        /* pointer not 16-byte aligned               */
  MOE_ERR_WORKSPACE = -4,        /* workspace missing or too small            */
  MOE_ERR_CUDA = -5              /* a CUDA runtime / driver call failed       */
};

enum moe_dtype { MOE_DTYPE_BF16 = 0, MOE_DTYPE_F32 = 1 };
enum moe_route_mode { MOE_ROUTE_TOPK = 0, MOE_ROUTE_RRE = 1 };
/* Expert network.  RELU: H = ReLU(x W1^T), out = H W2^T, W1 [E, f, d].
 * GEGLU (a gated linear unit in the feed-forward layer, "MosaicBERT" page:
 * the FFN uses GLU): W1 [E, 2f, d] whose rows 2i and 2i+1 are the gate and the
 * linear projection of hidden unit i, H_i = GELU(x . W1[2i]) * (x . W1[2i+1])
 * with GELU(a) = a * Phi(a) (the erf form), out = H W2^T; bf16 layers only. */
enum moe_expert { MOE_EXPERT_RELU = 0, MOE_EXPERT_GEGLU = 1 };
enum moe_status_bits {
  MOE_STATUS_TIMEOUT = 1,   /* a pipeline wait gave up (wait limit); outputs invalid  */
  MOE_STATUS_BAD_DOMAIN = 2, /* an RRE domain id was outside 0..G-1 (routed as 0)      */
  MOE_STATUS_BAD_COUNTS = 4, /* expert parallel: a row fell outside its expert's block
                                (counts that do not match the assignment); skipped     */
  MOE_STATUS_BAD_INDEX = 8   /* bounds-checked build only (moe_bounds_checked() == 1):
                                moe_dispatch / moe_combine met an expert index outside
                                0..E-1 or a slot outside 0..C-1; that choice skipped  */
};

/* One MoE layer.  56 bytes, no padding. */
typedef struct moe_config {
  int64_t T;          /* tokens in the batch (>= 0; T * k <= 2^31 - 1)                 */
  int32_t d_model;    /* token width d                                                 */
  int32_t d_ff;       /* expert hidden width f                                         */
  int32_t E;          /* experts, 1..256                                               */
  int32_t k;          /* experts per token: 1 or 2 (RRE: 1)                            */
  int32_t capacity;   /* C, tokens per expert (>= 0); see moe_capacity                 */
  int32_t mode;       /* enum moe_route_mode                                           */
  int32_t num_groups; /* RRE: G domain groups, E % G == 0; ignored for TOPK            */
  int32_t dtype;      /* enum moe_dtype of x, W_r, W1, W2, xe, H, ye, y                */
  int32_t expert;     /* enum moe_expert (0 = ReLU FFN)                                 */
  int32_t reserved;   /* must be 0                                                      */
  uint64_t seed;      /* RRE: seed of the splitmix64 routing hash; ignored for TOPK    */
} moe_config;

/* Workspace layout used by moe_layer_forward: byte offsets from the
 * workspace base (each 256-byte aligned) and the total size.  After a call
 * the caller may read any of these intermediate tensors. */
typedef struct moe_workspace_map {
  size_t logits;     /* [T, E] fp32 (fp32 TOPK layers only; bf16
                        layers fuse the gate into the router and
                        keep no logits: the region is empty)   */
  size_t expert_idx; /* [T, k] int32                            */
  size_t gate;       /* [T, k] fp32                             */
  size_t slot;       /* [T, k] int32                            */
  size_t kept;       /* [T, k] uint8                            */
  size_t tok_of_row; /* [E, C] int32, -1 where the slot is free */
  size_t arrivals;   /* [E] int32                               */
  size_t kept_cnt;   /* [E] int32                               */
  size_t n_dropped;  /* [1] int32                               */
  size_t scratch;    /* assignment scratch (moe_assign_workspace_size bytes) */
  size_t ffn_sync;   /* expert-FFN tile counters (moe_ffn_workspace_size bytes) */
  size_t xe;         /* [E, C, d] activations                   */
  size_t H;          /* [E, C, f] activations                   */
  size_t ye;         /* [E, C, d] activations                   */
  size_t total;
} moe_workspace_map;

/* ---- host-only queries (no CUDA call) --------------------------------- */

int32_t moe_abi_version(void);
/* sizeof(moe_config) and sizeof(moe_workspace_map) as compiled, for binders. */
size_t moe_config_size(void);
size_t moe_workspace_map_size(void);
/* Static text for an enum moe_error value. */
const char* moe_error_string(int32_t code);
/* Detail of the last error returned on the calling host thread ("" if none). */
const char* moe_last_error(void);

/* 1 if this library was built with bounds checks (MOE_CHECK_BOUNDS: the file
 * libmoe_b200_checked.so), else 0.  In that build moe_dispatch and
 * moe_combine check every expert index and slot they are given against E and
 * C before they touch a row, skip a choice that is out of range and report
 * it as MOE_STATUS_BAD_INDEX; the expert-parallel calls always check their
 * rows (MOE_STATUS_BAD_COUNTS).  A debugging aid for callers that build the
 * routing arrays themselves: the default build trusts them, as the layer's
 * own kernels produce them in range. */
int32_t moe_bounds_checked(void);

/* Limit of every bounded wait inside the library's kernels, in ns, for the
 * launches made after this call by any host thread (process-wide); 0
 * restores the default of 1 s.  For tests of the failure path and for
 * debugging: a wait that can never be met then ends within this limit and
 * the call reports MOE_STATUS_TIMEOUT.  moe_wait_limit_ns returns the value
 * in force. */
void moe_set_wait_limit_ns(uint64_t ns);
uint64_t moe_wait_limit_ns(void);

/* Eq. (3) of the Switch notes, sec. 2.2: floor(T / E * capacity_factor).
 * Returns -1 if E < 1, T < 0 or capacity_factor < 0. */
int32_t moe_capacity(int64_t T, int32_t E, double capacity_factor);

/* MOE_OK if `cfg` is a layer this library runs, else the error code. */
int32_t moe_config_check(const moe_config* cfg);

/* Bytes of scratch moe_topk_assign needs (0 if cfg is invalid).  The library's
 * assignment exchanges its counts on chip and needs none: 0 for every cfg. */
size_t moe_assign_workspace_size(const moe_config* cfg);

/* Bytes of scratch moe_expert_ffn needs (0 if cfg is invalid). */
size_t moe_ffn_workspace_size(const moe_config* cfg);

/* Layout (and total size) of the moe_layer_forward workspace. */
int32_t moe_workspace_layout(const moe_config* cfg, moe_workspace_map* out);
size_t moe_workspace_size(const moe_config* cfg); /* 0 if cfg is invalid */

/* Bytes of scratch moe_aux_loss needs (0 if cfg is invalid). */
size_t moe_aux_workspace_size(const moe_config* cfg);

/* Bytes of scratch sparseclip_norm needs for this many tensors. */
size_t sparseclip_workspace_size(int32_t n_dense, int32_t n_sparse);

/* ---- the layer, step by step ------------------------------------------ */

/* Router logits (Switch notes sec. 2.1; fp32 router per sec. 2.4):
 *   logits[t, e] = sum_c x[t, c] * Wr[e, c] (+ bias[e])
 * x [T, d] and Wr [E, d] in cfg->dtype; bias [E] fp32, nullable; logits
 * [T, E] fp32.  bf16 inputs: exact products, fp32 accumulation on the
 * tensor cores.  fp32 inputs: fp32 FMA chain. */
int32_t moe_router(const moe_config* cfg, const void* x, const void* Wr, const float* bias,
                   float* logits, int32_t* status, moe_stream_t stream);

/* Gate, expert choice and capacity-bounded slot assignment.
 * TOPK (Switch notes sec. 2.1 eq. 1, sec. 2.2 eq. 3): from logits [T, E]
 *   pick the k largest (ties -> lower expert index), gate[t, j] = the
 *   softmax probability of that expert over all E (no renormalisation).
 * RRE ("[Paper review] PanGu-Sigma", proposed method): from domain_id [T]
 *   (values 0..G-1) pick expert domain*(E/G) + splitmix64(seed, t) mod
 *   (E/G), gate 1.  logits unused (may be null).
 * Then, in token order (token t's choices before token t+1's), slot[t, j] =
 *   number of earlier choices of the same expert; kept[t, j] = slot < C;
 *   tok_of_row[e*C + s] = token in slot s of expert e, -1 if none;
 *   arrivals[e] = choices of e; kept_cnt[e] = min(arrivals[e], C);
 *   n_dropped[0] = sum_e max(0, arrivals[e] - C).
 * Outputs: expert_idx, slot [T, k] int32; gate [T, k] fp32; kept [T, k]
 * uint8; tok_of_row [E*C] int32; arrivals, kept_cnt [E] int32; n_dropped
 * [1] int32.  workspace: moe_assign_workspace_size(cfg) bytes (may be null
 * when that is 0). */
int32_t moe_topk_assign(const moe_config* cfg, const float* logits, const int32_t* domain_id,
                        int32_t* expert_idx, float* gate, int32_t* slot, uint8_t* kept,
                        int32_t* tok_of_row, int32_t* arrivals, int32_t* kept_cnt,
                        int32_t* n_dropped, void* workspace, size_t workspace_bytes,
                        int32_t* status, moe_stream_t stream);

/* Dispatch (the permutation the Switch router's dispatch tensor encodes,
 * sec. 2.4): xe[e, s, :] = x[t, :] for every kept choice (t, j) with
 * e = expert_idx[t, j], s = slot[t, j].  Rows of xe that no token fills are
 * left untouched.  x [T, d], xe [E, C, d] in cfg->dtype.  status: see
 * moe_bounds_checked (unused by the default build). */
int32_t moe_dispatch(const moe_config* cfg, const void* x, const int32_t* expert_idx,
                     const int32_t* slot, const uint8_t* kept, void* xe, int32_t* status,
                     moe_stream_t stream);

/* Expert FFNs as one grouped computation over the kept rows:
 *   H[e, r, :]  = round(ReLU(xe[e, r, :] . W1[e]^T))   W1 [E, f, d]
 *   ye[e, r, :] = round(H[e, r, :] . W2[e]^T)          W2 [E, d, f]
 * (cfg->expert == MOE_EXPERT_GEGLU: W1 [E, 2f, d] and H[e, r, i] =
 * round(GELU(xe[e, r, :] . W1[e, 2i]) * (xe[e, r, :] . W1[e, 2i + 1])))
 * for r < kept_cnt[e] (device int32 [E], values in 0..C).  xe, ye
 * [E, C, d] and H [E, C, f] (caller-provided scratch) in cfg->dtype; other
 * rows of H and ye are left untouched.  bf16 runs tcgen05 kernels with fp32
 * accumulation, chosen by the capacity: C <= 128, one persistent kernel for
 * both GEMMs (128 x 256 tiles); 128 < C < 512, two grouped launches (one per
 * GEMM, 128 x 256 tiles); C >= 512, SM pairs (cta_group::2): with
 * d_model >= 2048 one persistent kernel for both GEMMs (256 weight rows x up
 * to 256 tokens per tile), else two grouped launches (256 x 256 tiles).
 * workspace: moe_ffn_workspace_size bytes (zeroed by the call; the persistent
 * kernels' tile and dependency counters).  fp32 runs FMA GEMMs and may pass
 * a null workspace. */
int32_t moe_expert_ffn(const moe_config* cfg, const void* xe, const void* W1, const void* W2,
                       const int32_t* kept_cnt, void* H, void* ye, void* workspace,
                       size_t workspace_bytes, int32_t* status, moe_stream_t stream);

/* Flags of moe_expert_ffn_ex. */
enum moe_ffn_flags {
  /* The caller has already zeroed the workspace's moe_ffn_workspace_size
   * bytes earlier on `stream` (for example inside a kernel of its own), so
   * the call launches no memset and the persistent kernel reads its counters
   * as it finds them.  Its counters (uint32): word 0 numbers the tiles as
   * thread blocks take them; word 1 + e * ceil(C / 256) + c counts the
   * finished GEMM-1 work of rows chunk c of expert e (chunks of at most 256
   * rows; c = 0 when C <= 256), and the GEMM-2 tiles of that chunk wait
   * (bounded) until the count minus its total, as a signed 32-bit
   * difference, is >= 0.  A word preset to -n therefore ends n short and
   * that wait runs out. */
  MOE_FFN_WORKSPACE_ZEROED = 1
};

/* moe_expert_ffn with flags (enum moe_ffn_flags; 0 = moe_expert_ffn). */
int32_t moe_expert_ffn_ex(const moe_config* cfg, const void* xe, const void* W1, const void* W2,
                          const int32_t* kept_cnt, void* H, void* ye, void* workspace,
                          size_t workspace_bytes, uint32_t flags, int32_t* status,
                          moe_stream_t stream);

/* Combine (Switch notes sec. 2.1, eq. 2; drop rule sec. 2.2):
 *   y[t, :] = sum over kept j of gate[t, j] * ye[expert_idx[t, j], slot[t, j], :]
 * accumulated in fp32 and rounded once; 0 for a token with no kept choice.
 * y [T, d] in cfg->dtype. */
int32_t moe_combine(const moe_config* cfg, const void* ye, const int32_t* expert_idx,
                    const float* gate, const int32_t* slot, const uint8_t* kept, void* y,
                    int32_t* status, moe_stream_t stream);

/* The whole layer: router (TOPK) -> gate/top-k or RRE -> slot assignment ->
 * dispatch -> expert FFN -> combine, all on `stream`.  Wr (+ bias) for TOPK,
 * domain_id for RRE (the other may be null).  y [T, d] in cfg->dtype.
 * workspace: moe_workspace_size(cfg) bytes laid out as moe_workspace_layout
 * describes; it holds the intermediates after the call, except that bf16
 * layers fuse the gate into the router (no logits) and bf16 top-1 layers
 * fuse the combine into the expert FFN, which writes gate * E(x) straight
 * to y (ye is left untouched).
 * stage_events (nullable; a profiling hook): host array of 6 cudaEvent_t
 * (entries may be null) recorded on `stream` before the router and after
 * the router, the assignment, the dispatch, the expert FFN and the combine.
 * The call only enqueues work on `stream` (no host synchronisation, no
 * allocation), so it may be captured into a CUDA graph; the graph then
 * reads and writes the same buffers on every replay. */
int32_t moe_layer_forward(const moe_config* cfg, const void* x, const void* Wr, const float* bias,
                          const int32_t* domain_id, const void* W1, const void* W2, void* y,
                          void* workspace, size_t workspace_bytes, int32_t* status,
                          void* const* stage_events, moe_stream_t stream);

/* Switch auxiliary load-balancing loss and mean routing entropy (Switch
 * notes sec. 2.2, "A Differentiable Load Balancing Loss", eqs. (4)-(6); the
 * routing entropy the TorchScale review tracks), from router logits [T, E]
 * fp32 (moe_router's output; cfg->mode must be MOE_ROUTE_TOPK):
 *   p(x)   = softmax over all E experts of the token's logits (eq. 1)
 *   f[i]   = (1/T) #{tokens : argmax p = i}, ties to the lower index (eq. 5)
 *   P[i]   = (1/T) sum over tokens of p_i (eq. 6)
 *   out[0] = alpha * E * sum_i f[i] P[i]                                (eq. 4)
 *   out[1] = (1/T) sum over tokens of -sum_i p_i ln p_i
 * The pages use alpha = 1e-2.  out [2], f [E], P [E]: device double (f and P
 * nullable).  T = 0 gives zeros.  Softmax and entropy per token in fp32,
 * sums over tokens in double, added in a fixed order (deterministic).
 * workspace: moe_aux_workspace_size(cfg) bytes. */
int32_t moe_aux_loss(const moe_config* cfg, const float* logits, double alpha, double* out,
                     double* f, double* P, void* workspace, size_t workspace_bytes,
                     moe_stream_t stream);

/* SparseClip global gradient norm ("[Paper review] TorchScale", proposed
 * method): ||g||_2 = ||(g_d, kappa g_s)||_2 with kappa = 1/sqrt(num_experts),
 *   out[0] = sqrt(Sd + Ss / num_experts), out[1] = Sd, out[2] = Ss,
 *   Sd = sum of squares over the dense tensors, Ss over the expert tensors.
 * dense / sparse: host arrays of device fp32 pointers with host arrays of
 * element counts; out: device double[3].  Squares are summed in fp32 over
 * groups of 4 elements and in fp64 above that, in a fixed order, so the
 * result is the same on every run on the same GPU model.  n_dense + n_sparse
 * <= 4096.  workspace: sparseclip_workspace_size(n_dense, n_sparse) bytes. */
int32_t sparseclip_norm(const float* const* dense, const int64_t* dense_len, int32_t n_dense,
                        const float* const* sparse, const int64_t* sparse_len, int32_t n_sparse,
                        int32_t num_experts, double* out, void* workspace, size_t workspace_bytes,
                        moe_stream_t stream);

/* SparseClip clipping step (TorchScale review, proposed method: gradient
 * clipping by the reweighted L2 norm ||(g_d, kappa g_s)||_2, kappa = 1/sqrt(E)):
 * computes the norm exactly as sparseclip_norm (out[0..2]), then scales
 * every dense and expert tensor IN PLACE by
 *   coef = min(1, max_norm / norm)      (1 when norm <= max_norm: nothing written)
 * and writes coef to out[3].  kappa only reweights the norm; the same coef
 * applies to all tensors.  max_norm: positive, finite (the pages give no
 * value).  out [4] device double.  A tensor listed twice is scaled twice.
 * Same arguments, limits and workspace as sparseclip_norm otherwise; the
 * tensors are writable device fp32, 16-byte aligned. */
int32_t sparseclip_clip(float* const* dense, const int64_t* dense_len, int32_t n_dense,
                        float* const* sparse, const int64_t* sparse_len, int32_t n_sparse,
                        int32_t num_experts, double max_norm, double* out, void* workspace,
                        size_t workspace_bytes, moe_stream_t stream);

/* sparseclip_norm without a workspace, for callers that cannot allocate
 * device memory: a runtime whose HBM is handed out once at start-up by its
 * own pool and that forbids allocation afterwards, or code that must not call
 * the CUDA allocator where it runs (allocator callbacks, out-of-memory
 * recovery).  The pages describe no such entry point; it has no counterpart
 * there.  Same arguments and result as sparseclip_norm minus the workspace.
 * The partial sums live in a fixed 128 KiB array inside the library's own
 * device memory, present on every GPU that loads the library until the
 * process exits.  Limits and behaviour:
 *   * n_dense + n_sparse <= 1024, else MOE_ERR_UNSUPPORTED (nothing launched);
 *   * the first call with a device (and CUDA context) current looks up the
 *     array's device address and caches it per device and context, so a
 *     caller that switches contexts or resets the device gets a fresh
 *     lookup; make that first call before any stream capture;
 *   * the call allocates nothing (no cudaMalloc/cudaFree, no allocating
 *     library routine);
 *   * every call on a device shares the array: calls that overlap on the
 *     GPU (other streams or host threads) race, so the caller serialises
 *     them.  Each call writes every partial it reads, so no clearing is
 *     needed between calls. */
int32_t sparseclip_norm_noalloc(const float* const* dense, const int64_t* dense_len,
                                int32_t n_dense, const float* const* sparse,
                                const int64_t* sparse_len, int32_t n_sparse, int32_t num_experts,
                                double* out, moe_stream_t stream);

/* ---- expert parallelism over the GPUs of one node ---------------------- */

/* The sparse layer's distinct expert weights placed on different devices
 * (Switch notes sec. 2, opening paragraph: the parameter count grows with the
 * device count while each device's memory and compute stay bounded).
 * `world` ranks (1..8), El = E / world experts each: rank r holds experts
 * r*El .. (r+1)*El - 1 (W1, W2 shards [El, ...]).  Every rank routes and
 * assigns its own batch of cfg->T tokens exactly as moe_topk_assign does,
 * with capacity C = cfg->capacity per batch, so each rank's output equals the
 * single-device layer (moe_layer_forward) on that rank's batch.
 *
 * cnt_all [world, E] int32 (device): row q = the kept_cnt of rank q, exchanged
 * by the caller (an all-gather) before the dispatch.
 * Receive buffers: rank r's xe_r and ye_r are [El, world*C, d] in cfg->dtype.
 * The kept rows for its local expert el from rank q sit at rows
 * off_q(e) .. off_q(e) + cnt_all[q, e] - 1 of block el (e = r*El + el),
 * off_q(e) = sum over q' < q of cnt_all[q', e]: rank order, then slot order.
 *
 * One layer step on rank r:
 *   1. moe_router + moe_topk_assign on the rank's batch (global E);
 *   2. all-gather of kept_cnt into cnt_all;
 *   3. moe_ep_dispatch (stores rows into the home ranks' xe);
 *   4. a barrier across ranks (every rank's dispatch complete);
 *   5. moe_expert_ffn on xe_r with the config moe_ep_ffn_config gives and
 *      kept counts local_cnt, writing ye_r;
 *   6. a barrier across ranks (every rank's FFN complete);
 *   7. moe_ep_combine (loads rows from the home ranks' ye).
 * The library's kernels never wait on another rank: the caller's collectives
 * in steps 2, 4 and 6 order the ranks. */

/* The expert-FFN config of one rank: cfg with E = El, capacity = world*C
 * (k, mode and num_groups set to 1, TOPK and 1: routing does not enter the
 * FFN).  Host only.  MOE_ERR_INVALID_ARGUMENT if world is outside 1..8 or does
 * not divide E; MOE_ERR_UNSUPPORTED if world*C exceeds 2^31-1. */
int32_t moe_ep_ffn_config(const moe_config* cfg, int32_t world, moe_config* out);

/* Step 3.  For each kept choice (t, j) of this rank, with e = expert_idx[t, j],
 * h = e / El:  xe_h[e - h*El, off_rank(e) + slot[t, j], :] = x[t, :].
 * xe_peers: host array of `world` device pointers, entry q = rank q's xe as
 * mapped into this process (CUDA IPC or peer access; entry `rank` = this
 * rank's own), each 16-byte aligned.  local_cnt [El] int32 (device,
 * nullable): receives sum over q of cnt_all[q, rank*El + el], the kept counts
 * for step 5.  A row whose index would fall outside 0..world*C-1 is skipped
 * and sets MOE_STATUS_BAD_COUNTS.  x [T, d] in cfg->dtype.  Two launches: the
 * copy, then a one-thread kernel whose system-scope fence makes the copy's
 * stores visible to every device before the caller's next operation on
 * `stream` (the barrier of step 4). */
int32_t moe_ep_dispatch(const moe_config* cfg, int32_t rank, int32_t world, const void* x,
                        const int32_t* expert_idx, const int32_t* slot, const uint8_t* kept,
                        const int32_t* cnt_all, void* const* xe_peers, int32_t* local_cnt,
                        int32_t* status, moe_stream_t stream);

/* Step 7, the combine of eq. 2 (Switch notes sec. 2.1) over the home ranks'
 * outputs:  y[t, :] = sum over kept j of gate[t, j] *
 * ye_h[e - h*El, off_rank(e) + slot[t, j], :], fp32 accumulation in choice
 * order, one rounding; 0 for a token with no kept choice.  ye_peers: host
 * array of `world` device pointers as for moe_ep_dispatch.  y [T, d] in
 * cfg->dtype.  Out-of-block rows: skipped, MOE_STATUS_BAD_COUNTS. */
int32_t moe_ep_combine(const moe_config* cfg, int32_t rank, int32_t world,
                       const void* const* ye_peers, const int32_t* expert_idx, const float* gate,
                       const int32_t* slot, const uint8_t* kept, const int32_t* cnt_all, void* y,
                       int32_t* status, moe_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H_ */
