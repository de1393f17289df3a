/*
 * sfm.h -- C ABI of the performer's next-unit flow-matching denoising step
 * (Wan-Streamer v0.2) on one NVIDIA B200 (sm_100a).
 *
 * What the calls compute.  The pages describe the performer's per-unit work
 * without signatures: the thinker broadcasts a compact, performer-compatible
 * K/V slice; each performer rank writes it into a pre-allocated local cache;
 * the performer then runs the flow-matching solver over the next unit's audio
 * and video latents and returns them ("Wan-Streamer v0.2: Higher Resolution,
 * Same Latency" digest, "method overview and architecture"; "Wan-Streamer
 * v0.2" blog, "Infra"; v0.2 abstract).  The solver integrates the
 * rectified-flow path z_tau = (1 - tau) z0 + tau eps from tau = 1 to tau = 0
 * with Euler steps z <- z + (tau_next - tau) v, v = f_theta(z, tau | cache)
 * ("Wan-Streamer" v0.1 blog, §3.4 conditional flow matching), where f_theta is
 * the block-causal Transformer of §3.3: the current unit's tokens see every
 * cached unit and each other (bidirectional inside the unit).
 *
 * Conventions for every call:
 *   - Plain pointers.  "device" = CUDA device memory of the current device,
 *     "host" = ordinary host memory.  Matrices are row-major; a weight matrix
 *     W of a linear map x -> x W^T is stored [out][in].
 *   - stream: a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Calls are asynchronous on that stream: device buffers passed in must
 *     stay valid and unmodified until the stream has executed the call.
 *   - Every argument, session and capacity error is detected on the host
 *     BEFORE any launch and returned as a negative status; nothing is
 *     written in that case.  A CUDA launch failure returns SFM_ECUDA;
 *     asynchronous device errors surface on a later call.  No call aborts the
 *     process or throws across the ABI.
 *   - One handle is used by one host thread / one stream at a time.
 */
#ifndef SFM_H_
#define SFM_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SFM_API __attribute__((visibility("default")))
#else
#define SFM_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ------------------------------------------------------ */
#define SFM_OK             0
#define SFM_EINVAL        (-1)   /* bad argument (null pointer, size, shape)      */
#define SFM_ECAPACITY     (-2)   /* cache or pool full (ring off), batch too big  */
#define SFM_ESESSION      (-3)   /* session id not open                           */
#define SFM_ECUDA         (-4)   /* a CUDA call failed (see sfm_last_cuda_error)  */
#define SFM_ENOMEM        (-5)   /* device allocation failed in sfm_create        */
#define SFM_EUNSUPPORTED  (-6)   /* shape the kernels do not support              */
#define SFM_EDEVICE       (-7)   /* an earlier kernel of this handle gave up a
                                    bounded wait (see sfm_check_device_error);
                                    refused until sfm_clear_device_error        */

/* ---- storage / arithmetic type of weights, cache and activations -------- */
#define SFM_DTYPE_BF16 0   /* bf16 storage, tensor-core MMA with fp32 accumulation;
                              residual stream, softmax, z and v in fp32           */
#define SFM_DTYPE_FP32 1   /* fp32 everywhere (CUDA cores); small shapes          */

typedef struct sfm_handle sfm_handle;   /* opaque, library-owned */

/* Shapes of f_theta and of one streaming unit. */
typedef struct sfm_config {
  int n_layers;          /* L                                                   */
  int d_model;           /* d: multiple of 128 (bf16) / 64 (fp32)               */
  int n_heads;           /* H                                                   */
  int head_dim;          /* D_h: 128 for bf16; a multiple of 32, <= 128 for fp32 */
  int d_mlp;             /* F: multiple of 128 (bf16) / 64 (fp32)               */
  int c_lat;             /* C: latent channels per token (<= 64)                */
  int n_video;           /* video tokens of the current unit (raster order)     */
  int n_audio;           /* audio tokens of the current unit (after the video)  */
  int unit_kv_tokens;    /* T_u: K/V tokens the thinker sends per unit          */
  int max_sessions;      /* sessions open at once; also the largest batch       */
  long long pool_tokens; /* per-layer K/V rows of the cache pool shared by all
                            sessions; a session with capacity U units takes
                            U * T_u + (n_video + n_audio) rows                  */
  int dtype;             /* SFM_DTYPE_BF16 | SFM_DTYPE_FP32                     */
  int ring;              /* 1: a full session cache overwrites its oldest unit;
                            0: sfm_kvcache_append returns SFM_ECAPACITY          */
  double rope_theta;     /* RoPE base (10000)                                   */
  double rms_eps;        /* RMSNorm epsilon (1e-6)                              */
  /* Variants the pages leave open (the defaults, 0, are the plain readings). */
  int mlp;               /* SFM_MLP_GELU: x += GELU_tanh(h W_1^T) W_2^T, W_1 [F][d];
                            SFM_MLP_SWIGLU: x += (silu(h W_g^T) * (h W_u^T)) W_2^T,
                            W_1 [2F][d] holding W_g and W_u in interleaved blocks of
                            64 rows (rows 128 b + [0, 64): gate rows 64 b + [0, 64);
                            rows 128 b + [64, 128): the matching up rows); F % 64 == 0 */
  int rope;              /* SFM_ROPE_1D: positions p0 + j;
                            SFM_ROPE_3D: (t, y, x) per token -- t the unit's index on
                            the timeline (units appended before it), (y, x) the video
                            token's cell in a raster of grid_w columns, (0, 0) for
                            audio; the head's D/2 rotate-half pairs split into
                            D/2 - 2 (D/6) time pairs and D/6 pairs per spatial axis,
                            each axis with its own frequency ladder theta^(-k / n_axis) */
  int grid_w;            /* SFM_ROPE_3D: video raster width in tokens (>= 1)     */
} sfm_config;

#define SFM_MLP_GELU    0
#define SFM_MLP_SWIGLU  1
#define SFM_ROPE_1D     0
#define SFM_ROPE_3D     1

/*
 * Weights of f_theta: device pointers of the config's dtype, each 16-byte
 * aligned (else SFM_EINVAL), borrowed (not copied) for the handle's lifetime.  The per-layer members are HOST arrays
 * of n_layers device pointers; the arrays themselves are copied at create.
 *   w_in   [d][C]           x_j = W_in z_j + e_mod[m(j)] + temb(tau)
 *   e_mod  [2][d]           row 0 video, row 1 audio
 *   g_final[d], w_out[C][d] v = RMSNorm(x; g_final) W_out^T
 *   g_attn [d]              pre-attention RMSNorm gain
 *   w_qkv  [3 H D_h][d]     output rows: q (head-major, D_h per head), then k, then v
 *   w_o    [d][H D_h]
 *   g_mlp  [d]              pre-MLP RMSNorm gain
 *   w_1    [F][d], w_2 [d][F]   x += GELU_tanh(RMSNorm(x) W_1^T) W_2^T
 *                           (SwiGLU: w_1 [2F][d] in the interleaved layout above)
 * A handle created with w == NULL supports only the cache calls.
 */
typedef struct sfm_weights {
  const void* w_in;
  const void* e_mod;
  const void* g_final;
  const void* w_out;
  const void* const* g_attn;
  const void* const* w_qkv;
  const void* const* w_o;
  const void* const* g_mlp;
  const void* const* w_1;
  const void* const* w_2;
} sfm_weights;

/* Per-session cache bookkeeping (host copy). */
typedef struct sfm_session_info {
  int cache_units;          /* capacity in units (slots)                          */
  long long units_appended; /* units ever appended, evicted ones included         */
  long long valid_tokens;   /* min(units_appended, cache_units) * T_u             */
  long long p0;             /* position of the current unit's first token
                               = units_appended * T_u                             */
  long long base_row;       /* first pool row of this session                     */
} sfm_session_info;

/* ---- handle ------------------------------------------------------------- */

/* Validates cfg, allocates the K/V pool (2 * L * pool_tokens * H * D_h
 * elements) and all scratch on the current device.  Returns SFM_EINVAL /
 * SFM_EUNSUPPORTED for bad shapes, SFM_ENOMEM if allocation fails.  The hot
 * path allocates nothing after this call. */
SFM_API int sfm_create(const sfm_config* cfg, const sfm_weights* w, sfm_handle** out);

/* Frees everything the handle owns (synchronises the device first). */
SFM_API void sfm_destroy(sfm_handle* h);

/* Carves a contiguous cache region of cache_units unit slots (plus the
 * current unit's scratch rows) out of the pool for a new session.
 * SFM_ECAPACITY if the pool or the session table is full. */
SFM_API int sfm_session_open(sfm_handle* h, int cache_units, int* session);

/* Forgets a session's units (counters to zero); its region stays reserved. */
SFM_API int sfm_session_reset(sfm_handle* h, int session);

SFM_API int sfm_session_get_info(const sfm_handle* h, int session, sfm_session_info* out);

/* ---- the hot path ------------------------------------------------------- */

/*
 * Writes the thinker's K/V slice for n_tok / T_u whole units into the
 * session's cache ("Wan-Streamer v0.2" digest, "method overview and
 * architecture", performer path: each rank writes the broadcast, performer-
 * compatible K/V slice into its pre-allocated local cache; "Wan-Streamer v0.2"
 * blog, "Infra").  The pages state no eviction policy; here unit u
 * (u = units_appended + i) goes to slot u mod cache_units, rows verbatim.  k, v: device, [L][n_tok][H][D_h] of the
 * handle's dtype, caller-owned; K is already rotated (post-RoPE).
 * SFM_EINVAL if n_tok is not a positive multiple of T_u; SFM_ECAPACITY if
 * ring == 0 and the units do not fit (nothing is written).
 */
SFM_API int sfm_kvcache_append(sfm_handle* h, int session, const void* k, const void* v,
                       int n_tok, void* stream);

/*
 * sfm_kvcache_append for one rank of a head-sharded cache: the broadcast
 * slice's rows hold src_heads heads ([L][n_tok][src_heads][D_h]) and this
 * handle's cache keeps heads [head0, head0 + n_heads) of each, n_heads being
 * the handle's own head count ("Wan-Streamer v0.2" digest, "method overview
 * and architecture": each performer rank keeps a pre-sharded local cache and
 * writes the broadcast K/V slice into it; with Ulysses context parallelism a
 * rank attends over its own head group).  src_heads = n_heads, head0 = 0 is
 * sfm_kvcache_append.  SFM_EINVAL if the head range does not fit src_heads;
 * errors and ring behaviour otherwise as for sfm_kvcache_append.
 */
SFM_API int sfm_kvcache_append_heads(sfm_handle* h, int session, const void* k, const void* v,
                                     int n_tok, int src_heads, int head0, void* stream);

/* Copies cache rows [row0, row0 + n_rows) of one layer into caller device
 * buffers k_dst, v_dst ([n_rows][H][D_h]).  Rows index the session's region
 * (slot s occupies rows [s T_u, (s+1) T_u)). */
SFM_API int sfm_kvcache_read(const sfm_handle* h, int session, int layer, long long row0,
                     long long n_rows, void* k_dst, void* v_dst, void* stream);

/*
 * One Euler step of the current unit: v = f_theta(z, tau_from | cache),
 * z <- z + (tau_to - tau_from) v ("Wan-Streamer" v0.1 blog, §3.4 conditional
 * flow matching: the rectified-flow path and its velocity; §3.3: f_theta is the
 * block-causal Transformer, the unit seeing every cached unit and itself).  z: device fp32 [N][C], N = n_video +
 * n_audio (video rows first), updated in place.  v_out: nullable device fp32
 * [N][C] receiving v, a buffer other than z (SFM_EINVAL otherwise).  The
 * current unit's tokens are at positions p0 + j.
 */
SFM_API int sfm_denoise_step(sfm_handle* h, int session, float* z, float tau_from,
                     float tau_to, float* v_out, void* stream);

/*
 * The whole solve: Euler steps over taus[0] -> taus[1] -> ... -> taus[n-1]
 * (the performer's flow-matching solver for the next unit's audio and video
 * latents: "Wan-Streamer v0.2" digest, "method overview and architecture";
 * "Wan-Streamer" v0.1 blog, §3.4 and §5.1).  The pages give neither the step
 * count nor the schedule; the caller passes the schedule.
 * taus: host array, n_taus >= 2, taus[0] = 1 (z holds eps) decreasing to
 * taus[n-1] = 0 (z then holds the unit's clean latent).  The cache is not
 * modified (the current unit's K/V are scratch, never committed).
 */
SFM_API int sfm_fm_solve(sfm_handle* h, int session, float* z, const float* taus,
                 int n_taus, void* stream);

/* Batched solve over n_sessions open sessions (distinct ids), each with its
 * own cache length; z[i] is session i's device fp32 [N][C] (distinct buffers:
 * SFM_EINVAL if two entries are the same pointer).  sessions and z are host
 * arrays.  SFM_ECAPACITY if n_sessions > max_sessions. */
SFM_API int sfm_fm_solve_batched(sfm_handle* h, int n_sessions, const int* sessions,
                         float* const* z, const float* taus, int n_taus, void* stream);

/*
 * Classifier-free-guided solve, the sampler of the distillation teacher
 * ("Wan-Streamer" v0.1 blog, training, Stage 3: classifier-free guidance and
 * more flow-matching solver steps).  At every Euler step f_theta runs twice at
 * the same z and tau -- on `session` (the conditional context: the thinker's
 * K/V in its cache) and on `uncond_session` (the unconditional context) -- and
 * the step follows the guided velocity v = v_u + scale * (v_c - v_u), so
 * scale = 1 is the plain conditional solve and scale = 0 the unconditional
 * one.  The pages give no formula; this is the usual form of classifier-free
 * guidance.  The unconditional context is whatever uncond_session's cache
 * holds: a session with nothing appended (the unit attends to itself alone)
 * drops the condition entirely; one holding the K/V of a null prompt is the
 * other common choice.
 *   - z: device fp32 [N][C], updated in place (the one latent both
 *     evaluations read).  taus as for sfm_fm_solve.  Both evaluations write
 *     their unit's K/V into their own session's scratch rows, as a plain
 *     solve does; neither cache's contents or unit count change.
 *   - SFM_EINVAL if the two sessions are the same or scale is not finite.
 *   - Runs as one batch of two evaluations: needs max_sessions >= 2
 *     (SFM_ECAPACITY otherwise).
 */
SFM_API int sfm_fm_solve_guided(sfm_handle* h, int session, int uncond_session, float* z,
                                const float* taus, int n_taus, float scale, void* stream);
/*
 * n_pairs guided solves in one batch of 2 * n_pairs evaluations.  sessions,
 * uncond_sessions, z: host arrays of n_pairs entries (z[p] device fp32
 * [N][C], distinct buffers); all 2 * n_pairs session ids distinct.  v_out:
 * NULL, or a host array of n_pairs device fp32 [N][C] buffers (entries may be
 * NULL; non-NULL ones distinct, none of them a z) that receive the guided
 * velocity of the last step.  SFM_EINVAL if a z or v_out buffer repeats.  SFM_ECAPACITY if
 * 2 * n_pairs > max_sessions.
 */
SFM_API int sfm_fm_solve_guided_batched(sfm_handle* h, int n_pairs, const int* sessions,
                                        const int* uncond_sessions, float* const* z,
                                        const float* taus, int n_taus, float scale,
                                        float* const* v_out, void* stream);

/*
 * Velocities of several consecutive units in one pass of f_theta under the
 * general block-causal mask ("Wan-Streamer" v0.1 blog, §3.3: a unit sees
 * itself bidirectionally and every earlier unit, never a later one), the pass a
 * multi-unit prefill needs (the v0.2 blog's project-page note: a scene goes live
 * about 0.5 s after its prompt, thinker and performer prefill included).
 *   - The n_units units follow the session's cache on the timeline: token j of
 *     unit u is at position p0 + u N + j and sees every valid cached token,
 *     every token of units <= u and no token of a later unit.  One unit gives
 *     sfm_denoise_step's velocity.
 *   - z: host array of n_units device fp32 [N][C] latents (read only), unit u
 *     at flow time taus[u] (host array).  v_out: host array of n_units distinct
 *     device fp32 [N][C] buffers (none of them a z) receiving the velocities.
 *   - commit = 1 appends the units' own K/V, as computed in this pass (at their
 *     flow times; clean units have tau = 0), to the session's cache as n_units
 *     units.  Needs unit_kv_tokens == N (SFM_EUNSUPPORTED) and n_units free
 *     slots (the ring does not wrap here: SFM_ECAPACITY).  commit = 0 changes
 *     no cache state: the pass's K/V are scratch rows.
 *   - SFM_ECAPACITY if n_units > max_sessions (activation scratch) or if the
 *     pass's rows do not fit the session's region: valid_tokens + n_units N <=
 *     cache_units T_u + N.
 */
SFM_API int sfm_velocity_units(sfm_handle* h, int session, int n_units, const float* const* z,
                               const float* taus, float* const* v_out, int commit, void* stream);

/*
 * Launch mode of sfm_denoise_step / sfm_fm_solve / sfm_fm_solve_batched.
 * enabled = 1 (the default): each call is captured into one CUDA graph on a
 * stream private to the handle and the graph is launched on the caller's
 * stream (the handle keeps the executable graph and updates it in place on
 * the next call).  enabled = 0: kernels are launched directly on the
 * caller's stream.  Results are identical in both modes.  A call made while
 * sfm_profile_begin is in effect launches directly (the profiler brackets
 * every launch with events).  SFM_EINVAL for other values.  No counterpart
 * in the method's description: a launch mechanism.
 */
SFM_API int sfm_set_graph_mode(sfm_handle* h, int enabled);

/* ---- standalone kernels --------------------------------------------------- */

/*
 * Softmax attention O = softmax(Q K^T / sqrt(D_h)) V per head, every key
 * visible to every query (the performer form of block-causal attention: all
 * keys are cached units <= the current one or the current unit itself).
 * q: [n_q][H][D_h], k, v: [n_kv][H][D_h], o: [n_q][H][D_h], device, dtype as
 * given.  workspace: device scratch of at least
 * sfm_attention_workspace_bytes(...) bytes (caller-owned; may be NULL when
 * that size is 0).  n_kv >= 1.
 */
SFM_API size_t sfm_attention_workspace_bytes(int n_q, int n_kv, int n_heads, int head_dim, int dtype);
SFM_API int sfm_attention(const void* q, const void* k, const void* v, void* o, int n_q, int n_kv,
                  int n_heads, int head_dim, int dtype, void* workspace,
                  size_t workspace_bytes, void* stream);

/*
 * General block-causal attention ("Wan-Streamer" v0.1 blog, §3.3: a unit sees
 * itself bidirectionally and every earlier unit, never a later one), the form
 * a multi-unit pass such as a scene prefill needs.  The n_q queries are
 * n_q / unit_tokens units of unit_tokens tokens (the last one may be shorter);
 * the last n_q of the n_kv keys are theirs, in the same order, and the first
 * n_kv - n_q keys are a prefix (earlier context, e.g. a cache) every query
 * sees.  Query i attends to keys [0, n_kv - n_q + min((i / unit_tokens + 1) *
 * unit_tokens, n_q)).  unit_tokens >= n_q gives sfm_attention's result (every
 * key visible).  Layouts, dtypes, workspace (same size as for sfm_attention)
 * and errors as for sfm_attention; SFM_EINVAL if unit_tokens < 1 or
 * n_kv < n_q.  Key tiles past a query block's last visible key are skipped,
 * so the causal half of the work is not done.
 */
SFM_API int sfm_attention_block_causal(const void* q, const void* k, const void* v, void* o,
                                       int n_q, int n_kv, int unit_tokens, int n_heads,
                                       int head_dim, int dtype, void* workspace,
                                       size_t workspace_bytes, void* stream);

/*
 * sfm_attention without any allocation.  No counterpart in the paper: this
 * entry point exists for callers that cannot allocate device memory where they
 * need attention -- a real-time serving loop with a hard per-unit deadline
 * (cudaMalloc / cudaFree may synchronise the device and stall it), or a host
 * program whose own allocator owns all device memory.
 *   - Same arguments and result as sfm_attention, minus the workspace: the
 *     split-KV partials live in a fixed array of SFM_NOALLOC_SCRATCH_BYTES
 *     compiled into the library, which every GPU that loads the library holds
 *     until the process exits.  The call allocates and frees nothing.
 *   - Returns SFM_ECAPACITY, launching nothing, when the shape needs more
 *     scratch than that (sfm_attention_workspace_bytes(...) is the need).
 *   - The first call on each device resolves the array's device address with
 *     that device current (cudaGetSymbolAddress) and keeps it for that
 *     device's context (after a cudaDeviceReset the next call resolves it
 *     again); make that first call before any stream capture.
 *   - A bounded wait that gives up inside the kernel is reported through
 *     sfm_check_call_error, as for the other standalone calls.
 *   - Every call shares the one array per device, and it keeps the last call's
 *     contents (nothing in it needs to start at zero).  Calls that overlap on
 *     the GPU -- on different streams or from different threads -- race on it:
 *     order them on one stream.
 */
#define SFM_NOALLOC_SCRATCH_BYTES (64u << 20)
SFM_API int sfm_attention_noalloc(const void* q, const void* k, const void* v, void* o, int n_q,
                                  int n_kv, int n_heads, int head_dim, int dtype, void* stream);

/*
 * One dense projection of f_theta, y = x W^T: x [M][K], w [N][K] (device,
 * dtype as given), y [M][N].  epilogue: SFM_LINEAR_F32 writes fp32 y;
 * SFM_LINEAR_OUT writes y in dtype; SFM_LINEAR_GELU writes GELU_tanh(x W^T) in
 * dtype; SFM_LINEAR_RESID adds x W^T to an fp32 y in place (the residual
 * stream).  bf16: N a multiple of 128, K of 64 (tcgen05 tensor cores);
 * fp32: N a multiple of 64, K of 16 (CUDA cores).
 */
#define SFM_LINEAR_F32   0
#define SFM_LINEAR_OUT   1
#define SFM_LINEAR_GELU  2
#define SFM_LINEAR_RESID 3
SFM_API int sfm_linear(const void* x, const void* w, void* y, int M, int N, int K, int epilogue,
                       int dtype, void* stream);

/* Vectorised Euler update z[i] += dtau * v[i], i < n; device fp32. */
SFM_API int sfm_euler_update(float* z, const float* v, float dtau, long long n, void* stream);

/*
 * Test-only closed-form check of the solve loop: the Euler solve of
 * sfm_fm_solve with f_theta replaced by the exact velocity of the rectified-
 * flow path ("Wan-Streamer" v0.1 blog, §3.4: z_tau = (1 - tau) z0 + tau eps,
 * constant velocity eps - z0), written as the state-dependent (z - z0) / tau
 * and evaluated at each step's starting tau.  From z = eps at taus[0] = 1 any
 * schedule ends at z0 (up to fp32 rounding); a step that evaluated the velocity
 * at its end point, or moved the wrong way, would not.  z0, z: device fp32
 * [N][C] (N, C of the handle's configuration); z updated in place.  taus: host,
 * n_taus >= 2, finite, every tau but the last > 0 (SFM_EINVAL otherwise).
 * Uses no session and no weights.
 */
SFM_API int sfm_fm_solve_exact_velocity(const sfm_handle* h, const float* z0, float* z,
                                        const float* taus, int n_taus, void* stream);

/* ---- measurement ------------------------------------------------------------ */
/* Kernel classes timed by the profiler (index into the arrays below). */
#define SFM_PROF_APPEND     0   /* K/V cache append                          */
#define SFM_PROF_ATTN       1   /* attention (flash kernel)                  */
#define SFM_PROF_ATTN_MERGE 2   /* split-KV merge                            */
#define SFM_PROF_GEMM_QKV   3   /* QKV projection                            */
#define SFM_PROF_GEMM_O     4   /* O projection + residual                   */
#define SFM_PROF_GEMM_UP    5   /* MLP up + GELU                             */
#define SFM_PROF_GEMM_DOWN  6   /* MLP down + residual                       */
#define SFM_PROF_ROWOPS     7   /* embed, RMSNorm, RoPE, scatter, tables     */
#define SFM_PROF_HEAD       8   /* velocity head + Euler update              */
#define SFM_PROF_KINDS      9

/* Starts recording a CUDA event pair around every kernel this library
 * launches on this host thread (events on the launching stream), for up to
 * max_launches launches; later launches are not recorded.  Allocates the
 * events (not on the hot path).  SFM_EINVAL if max_launches < 1. */
SFM_API int sfm_profile_begin(int max_launches);
/* Synchronises the recorded events, stops recording and returns, per kernel
 * class, the summed device time in ms and the launch count (host arrays of
 * SFM_PROF_KINDS entries). */
SFM_API int sfm_profile_end(double* ms, long long* launches);
/* Kernels launched by this library in this process so far. */
SFM_API unsigned long long sfm_kernel_launch_count(void);

/* ---- errors --------------------------------------------------------------- */
/*
 * Bounded waits.  Every wait inside the tensor-core kernels (on a TMA load, an
 * MMA, or another role of the CTA) gives up after a bound (1 s): the waiting
 * role records its wait site in an error word, the CTA's roles unwind (drain
 * their own asynchronous copies with bounded waits, free tensor memory, write
 * zeros for the rows they own) and the kernel returns, so the CUDA context
 * stays usable.  Results of a call in which a wait gave up are invalid.
 *
 * Handle calls.  sfm_check_device_error synchronises the device and returns
 * the handle's word in *code: 0 when no kernel of the handle gave up, else the
 * site (0x1nn: a projection kernel, 0x2nn: the attention kernel; nn names the
 * wait).  Each solve also copies the word to host memory when it ends, so once
 * that copy has executed, every f_theta call on the handle (sfm_denoise_step,
 * sfm_fm_solve*, sfm_velocity_units) returns SFM_EDEVICE without launching,
 * until sfm_clear_device_error (which synchronises the device and zeroes both).
 *
 * Standalone calls (sfm_attention*, sfm_linear) share one word per device:
 * sfm_check_call_error synchronises the current device, returns that word in
 * *code and zeroes it.
 */
SFM_API int sfm_check_device_error(const sfm_handle* h, int* code);
SFM_API int sfm_clear_device_error(sfm_handle* h);
SFM_API int sfm_check_call_error(int* code);

/*
 * Test-only fault injection for the bounded waits (no counterpart in the
 * method: it exercises the failure path without faulting the GPU).  From the
 * next launch on, the kernels of handle h (h == NULL: the standalone calls of
 * this process) run with the given fault bits and wait bound:
 *   SFM_FAULT_ATTN_NO_LOADS  the attention kernel's TMA producer issues no loads,
 *   SFM_FAULT_GEMM_NO_LOADS  the projection kernels' TMA producers issue none,
 * so the roles that wait for those loads give up after wait_ns nanoseconds and
 * the kernel unwinds.  wait_ns = 0 restores the 1 s bound; otherwise 1e4 <=
 * wait_ns <= 1e10 (SFM_EINVAL outside, or for unknown fault bits).  faults = 0
 * and wait_ns = 0 restore normal operation.
 */
#define SFM_FAULT_NONE           0
#define SFM_FAULT_ATTN_NO_LOADS  1
#define SFM_FAULT_GEMM_NO_LOADS  2
SFM_API int sfm_test_fault(sfm_handle* h, int faults, long long wait_ns);

/*
 * The launch plan a handle fixed at create for its four projections (index 0
 * QKV, 1 O, 2 MLP-up, 3 MLP-down), chosen for a full batch of max_sessions
 * units: N-tile width, whether the projection runs on CTA pairs
 * (tcgen05 cta_group::2, 256-row tiles), and its K slices (1 = none).
 * fused_norm = 1 when every RMSNorm is split between the kernel that updates
 * the residual (it writes bf16(x g) and partial sums of squares) and the next
 * projection (bf16 handles).  No counterpart in the method: introspection.
 */
typedef struct sfm_plan {
  int block_n[4];
  int pair[4];
  int k_splits[4];
  int fused_norm;
} sfm_plan;
SFM_API int sfm_get_plan(const sfm_handle* h, sfm_plan* out);

/*
 * The key-range split counts the tcgen05 attention of a batched f_theta call
 * uses (introspection, no counterpart in the method).  n_sessions sessions of
 * rows_per_session query rows each, session i attending to n_keys[i] keys (its
 * cached tokens plus the current unit), n_heads heads, on a device of sms SMs:
 * splits[i] (host memory, n_sessions entries, caller-owned) receives session i's
 * count in [1, 16].  A session of one split has its output written by the
 * attention kernel itself; the others' partial results are merged.  Host only
 * (no device work).  SFM_EINVAL if a pointer is NULL, n_sessions is outside
 * [1, 16], or rows_per_session, n_heads, sms or an n_keys[i] is < 1.
 */
SFM_API int sfm_attention_batch_splits(int n_sessions, int rows_per_session, const long long* n_keys,
                                       int n_heads, int sms, int* splits);
SFM_API const char* sfm_strerror(int status);
/* The cudaError_t of the last failed CUDA call made by this library on this
 * host thread (0 if none). */
SFM_API int sfm_last_cuda_error(void);

#ifdef __cplusplus
}
#endif
#endif /* SFM_H_ */
