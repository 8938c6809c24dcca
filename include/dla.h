/*
 * dla.h -- C ABI of libdla.so, the B200 (sm_100a) Dynamic Linear Attention
 * (DLA) forward.
 *
 * The method ("Dynamic Linear Attention | Chlience Paper Archive", sections
 * 5.1-5.3; ai-feeds.com "Dynamic Linear Attention" summary, section 方法):
 * each token writes v_t phi(k_t)^T into the open segment state; a token joins
 * the open segment only when its score r_t = 1 - cos(k_t, k_{t-1}) and its
 * predecessor's are both below tau, otherwise it opens a new state; at most C
 * states (open one included) are kept in time order by merging the adjacent
 * sealed pair with the smallest Ward loss n_i n_j/(n_i+n_j) |mu_i - mu_j|^2
 * (mu = mean phi(k), leftmost on ties, merged state keeps the earlier
 * timestamp); the output is o_t = sum_i lambda_{t,i} S_i phi(q_t) with
 * lambda_{t,i} = softmax_i(phi(q_t) . mu_i / sqrt(d_k)).  phi = elu + 1.
 *
 * Conventions for every entry point:
 *   - All tensor arguments are DEVICE pointers to caller-owned memory; the
 *     library allocates no device memory and keeps no state between calls
 *     (apart from the scratch of dla_decode_step_static, below).
 *   - Every call is enqueued on `stream` (a cudaStream_t passed as void*;
 *     NULL = legacy default stream) and returns without synchronising.  A
 *     prefill forks its kernels onto auxiliary non-blocking streams (created
 *     on first use, once per host thread and device) with events recorded on
 *     `stream`, and joins back on `stream`: later work on `stream` sees all
 *     of its results, as if every kernel had run there.
 *   - Argument errors are returned synchronously (nothing is enqueued).
 *   - Errors found on the device (trace overflow, broken invariant) are
 *     written to *dev_status (a device int32 the caller zeroes beforehand and
 *     reads after synchronising); the first error code wins.
 *   - Calls are reentrant; concurrent calls must not share a cache, trace,
 *     workspace or dev_status.
 *   - Layouts are row-major with the last index fastest.  q, k, v are
 *     [B][H][T][d]; o is [B][H][T][d_v] in the input dtype (fp32 accumulation).
 *     Prefill tensors must start on a 16-byte boundary.
 */
#ifndef DLA_H_
#define DLA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  DLA_OK = 0,
  DLA_ERR_INVALID_ARG = 1,     /* null pointer, bad size, mismatched shapes */
  DLA_ERR_UNSUPPORTED = 2,     /* d_k != d_v, d not in {32, 64, 128}, C < 2; on the device:
                                  a cache the policy cannot continue */
  DLA_ERR_CUDA = 3,            /* a CUDA launch failed (see cudaGetLastError) */
  DLA_ERR_TRACE_OVERFLOW = 4,  /* device: more merges than dla_trace.cap */
  DLA_ERR_WORKSPACE = 5,       /* ws_bytes smaller than the size query */
  DLA_ERR_INVARIANT = 6,       /* device: a cache invariant was violated */
  DLA_ERR_TIMEOUT = 7,         /* device: a bounded wait inside a kernel gave up */
  DLA_ERR_CAPACITY = 8         /* device: the unbounded policy ran out of cache slots */
} dla_status;

/* Most state slots a cache may have (the unbounded policy's storage; the
 * capacity-bounded policies take 2 <= C <= 128). */
#define DLA_MAX_SLOTS 1024

typedef enum { DLA_F32 = 0, DLA_BF16 = 1 } dla_dtype;

typedef enum {
  DLA_POLICY_DYNAMIC = 0,   /* cosine score, capacity C, Ward merges (dla_prefill) */
  DLA_POLICY_FENWICK = 1,   /* fixed Fenwick buckets (dla_fixed_policy_prefill) */
  DLA_POLICY_INFO = 2,      /* the pages' state score and density merges */
  DLA_POLICY_UNBOUNDED = 3  /* DLA(I): cosine score, no capacity bound (dla_unbounded_prefill) */
} dla_policy;

/* Kernel kinds reported through dla_profile. */
typedef enum {
  DLA_K_SCORE = 0,       /* score + boundary scan */
  DLA_K_SEGSCAN = 1,     /* window piece scan */
  DLA_K_SEGSUM = 2,      /* fp64 piece sums of phi(k) */
  DLA_K_ENGINE = 3,      /* capacity-merge engine / bucket planner */
  DLA_K_MATERIALIZE = 4, /* state build, merges and versions */
  DLA_K_READOUT = 5,     /* multi-state readout */
  DLA_K_DECODE_DECIDE = 6,
  DLA_K_DECODE_STREAM = 7,
  DLA_K_BUILD = 8,       /* tensor-core state-piece builder */
  DLA_K_READOUT_PRE = 9, /* tensor-core readout prologue (weights, intra-tile output) */
  DLA_K_PHI = 10,        /* phi(q) as the bf16 tensor-core operand */
  DLA_K_INFO_SCORE = 11  /* information policy: state score + boundary */
} dla_kernel_kind;

/* Optional timing hook (host memory, caller-owned).  When non-NULL, the
 * library records begin[i] / end[i] (cudaEvent_t handles created by the
 * caller) on the launch stream around the i-th kernel it launches, stores its
 * dla_kernel_kind in kind[i] and advances `count`; launches past `cap` are not
 * recorded.  It adds two event records per launch and changes no result. */
typedef struct {
  void **begin, **end;
  int32_t *kind;
  int32_t cap, count;
} dla_profile;

/* One prefill call.  d_k == d_v in {32, 64, 128}.  C >= 2 is the cache
 * capacity (ignored by the fixed policy).  `window` = tokens per internal
 * window (multiple of 128; 0 = library default); it changes memory use and
 * speed, never results. */
typedef struct {
  int32_t B, H, T, d_k, d_v, C;
  float tau;
  int32_t in_dtype; /* dla_dtype of q, k, v and o */
  int32_t window;
  dla_profile *profile; /* optional timing hook, NULL in normal use */
} dla_config;

/* The DLA state cache of N sequences x H heads (device memory, caller-owned,
 * laid out by dla_cache_init inside one buffer).  It is the capacity-bounded
 * memory M = {(S_i, n_i, ...)} of Chlience section 5.2; prefill leaves it
 * ready for decode and a prefill on a non-empty cache continues the sequence.
 * States live in slots; `order` lists the live slots in time order, the last
 * one being the open state.  Per (n, h) = u:
 *   S         float  [u][C][d_v][d_k]  slot states sum v phi(k)^T (fp32)
 *   z         double [u][C][d_k]       slot sums of phi(k) (fp64, decisions)
 *   n, ts     int64  [u][C]            token count and first token of a slot
 *   pair_loss double [u][C]            Ward loss of sealed pair (p, p+1); entry
 *                                      C-1 (no pair) is -1 after the
 *                                      information policy, -2 after the
 *                                      unbounded one, 0 otherwise
 *   order     int32  [u][C]            time-order position -> slot
 *   m         int32  [u]               live states (open one included)
 *   prev_k    float  [u][d_k]          last key, for the next score
 *   prev_r    double [u]               last score
 *   t         int64  [u]               tokens seen                          */
typedef struct {
  int32_t N, H, C, d_k, d_v;
  float *S;
  double *z;
  int64_t *n, *ts;
  double *pair_loss;
  int32_t *order;
  int32_t *m;
  float *prev_k;
  double *prev_r;
  int64_t *t;
} dla_cache;

/* Optional decision trace of one prefill call (device memory):
 *   boundary    uint8 [B*H][T]   1 where token t opened a state
 *   merge_t     int32 [B*H][cap] global token index of each merge
 *   merge_i     int32 [B*H][cap] 0-based time-order position of the merged
 *                                pair's left member among sealed states
 *   merge_count int32 [B*H]      merges (may exceed cap: overflow status)  */
typedef struct {
  uint8_t *boundary;
  int32_t *merge_t, *merge_i, *merge_count;
  int32_t cap;
} dla_trace;

/* Bytes of device memory a cache of this shape needs (256-byte aligned). */
size_t dla_cache_bytes(int32_t N, int32_t H, int32_t C, int32_t d_k, int32_t d_v);

/* Lay out a cache in [dev_base, dev_base + bytes) and reset it to the empty
 * state (m = 0, t = 0, prev_r = 0; every array but S zeroed) with an
 * asynchronous memset on `stream`.  S is left as it is: a slot's state is
 * always written (new open state, store, merge) before it is read.
 * dev_base must be 256-byte aligned. */
dla_status dla_cache_init(dla_cache *cache, int32_t N, int32_t H, int32_t C, int32_t d_k,
                          int32_t d_v, void *dev_base, size_t bytes, void *stream);

/* Workspace bytes for dla_prefill (policy = DLA_POLICY_DYNAMIC),
 * dla_fixed_policy_prefill (DLA_POLICY_FENWICK) or dla_info_policy_prefill
 * (DLA_POLICY_INFO) with this config; 0 for an invalid config or policy. */
size_t dla_workspace_bytes(const dla_config *cfg, int32_t policy);

/* DLA prefill of T tokens for B x H streams, continuing `cache` (required,
 * B == cache->N, H == cache->H, same C, d).  Writes o [B][H][T][d_v] and,
 * when `trace` is non-NULL, the decision trace.  ws: device workspace of at
 * least dla_workspace_bytes(cfg, DLA_POLICY_DYNAMIC) bytes. */
dla_status dla_prefill(const dla_config *cfg, const void *q, const void *k, const void *v,
                       void *o, const dla_cache *cache, const dla_trace *trace, void *ws,
                       size_t ws_bytes, int32_t *dev_status, void *stream);

/* Workspace bytes for dla_decode_step on a cache of this shape. */
size_t dla_decode_workspace_bytes(int32_t N, int32_t H, int32_t C, int32_t d_k, int32_t d_v);

/* One token for each of the N x H streams of `cache`: decision, any capacity
 * merge, state write and readout; equivalent to dla_prefill with T = 1.
 * q, k, v [N][H][d] and o [N][H][d_v] in `in_dtype`.  Optional outputs:
 * boundary [N][H] (uint8) and merge_i [N][H] (int32, -1 = no merge).
 * profile: optional timing hook (NULL in normal use). */
dla_status dla_decode_step(const dla_cache *cache, float tau, int32_t in_dtype,
                           const void *q, const void *k, const void *v, void *o,
                           uint8_t *boundary, int32_t *merge_i, void *ws, size_t ws_bytes,
                           int32_t *dev_status, void *stream, dla_profile *profile);

/* dla_decode_step for callers that cannot allocate device memory: runtimes
 * that own a fixed device-memory budget, plug-ins that run inside another
 * engine's memory pool, or code paths where an allocation call is not
 * allowed.  Same arguments and results as dla_decode_step minus the
 * workspace: its scratch is a library-owned static device array of 8 MiB
 * (DLA_STATIC_DECODE_MAX_BYTES) that every GPU loading the library keeps until
 * the process exits.  It accepts caches whose dla_decode_workspace_bytes() is
 * at most that size (about 30,000 streams at C = 64) and returns
 * DLA_ERR_WORKSPACE for larger ones.  It allocates nothing.  The first call on
 * a device looks up the array's device address (cudaGetSymbolAddress) with
 * that device current; make that first call before any stream capture.  The
 * address is kept with the id of the context it was found in: after a
 * cudaDeviceReset or any other context teardown, the next call on the device
 * looks it up again, so that call too must come before any capture.  All
 * calls share the one array and it keeps the last call's contents (every call
 * rewrites what it reads, so nothing needs clearing); calls that overlap on
 * the GPU, from any stream or thread, race on it, so serialise them.  The
 * pages describing the method have no counterpart of this entry point. */
#define DLA_STATIC_DECODE_MAX_BYTES ((size_t)8 << 20)
dla_status dla_decode_step_static(const dla_cache *cache, float tau, int32_t in_dtype,
                                  const void *q, const void *k, const void *v, void *o,
                                  uint8_t *boundary, int32_t *merge_i, int32_t *dev_status,
                                  void *stream);

/* The Log-Linear-style fixed policy through the same engine (Chlience
 * section 2 and section 5.4): token t reads the Fenwick blocks of [0, t-1]
 * (one per set bit of t) plus {t}, with the same softmax over block means.
 * Starts every stream at t = 0; cfg->C and cfg->tau are ignored. */
dla_status dla_fixed_policy_prefill(const dla_config *cfg, const void *q, const void *k,
                                    const void *v, void *o, void *ws, size_t ws_bytes,
                                    int32_t *dev_status, void *stream);

/* The pages' own decision and merge rule (Chlience section 5.1 and section
 * 5.2) through the same windows, engine and readout as dla_prefill:
 *   - token t's state v_t phi(k_t)^T is compared with the open state S after
 *     RMSNorm over all d_v x d_k entries (no gain):
 *       I_t = |N(v_t phi(k_t)^T) - N(S)|_F / (|N(S)|_F + 1e-6),
 *       N(X) = X / sqrt(mean of X^2 + 1e-6);
 *   - I_t >= tau opens a new state; the first token of a stream opens one
 *     with I = 0;
 *   - each state keeps the sum of its tokens' scores, and at capacity the
 *     adjacent sealed pair with the least (sum_i + sum_i+1) / (n_i + n_i+1)
 *     merges (leftmost on ties); the readout is dla_prefill's.
 * Arguments as for dla_prefill; ws: at least dla_workspace_bytes(cfg,
 * DLA_POLICY_INFO) bytes.  The decisions need the open state in fp64 and the
 * states' score sums, which the cache does not hold, so every stream starts
 * from an empty cache: a stream whose cache has t > 0 sets
 * DLA_ERR_UNSUPPORTED in *dev_status and its outputs are unspecified.  After
 * the call the cache holds the policy's states, counts and time order, and
 * pair_loss the pair densities, with its unused last entry set to -1 to mark
 * the cache as this policy's: dla_prefill, dla_decode_step and
 * dla_decode_step_static (cosine score, Ward merges) set DLA_ERR_UNSUPPORTED
 * in *dev_status on such a stream, and its results are unspecified, until
 * dla_cache_init resets the cache. */
dla_status dla_info_policy_prefill(const dla_config *cfg, const void *q, const void *k,
                                   const void *v, void *o, const dla_cache *cache,
                                   const dla_trace *trace, void *ws, size_t ws_bytes,
                                   int32_t *dev_status, void *stream);

/* DLA(I), dynamic merging without the capacity bound (the ablation row
 * "Mamba-2 + DLA(I)" of the Chlience page's ablation table): the decisions of
 * dla_prefill (cosine score, two consecutive low scores join a token to the
 * open state) with no capacity merge at all.  Every segment stays a state of
 * its own and the readout's softmax runs over all of them, so the state count
 * grows with the sequence.  cfg->C is the cache's number of slots (storage
 * only, 2 <= C <= DLA_MAX_SLOTS; on the fp32 SIMT path, used for inputs
 * other than bf16 at d = 128, a tile's C logits must also fit in shared
 * memory, else DLA_ERR_UNSUPPORTED).  A stream that needs more states than C
 * sets DLA_ERR_CAPACITY in *dev_status; its later boundaries are then not
 * opened and its results are unspecified.  The cache must be empty or hold
 * a stream of this policy (a call continues it); a stream of another policy
 * sets DLA_ERR_UNSUPPORTED and its results are unspecified.  Afterwards pair_loss[C-1] is -2, which dla_prefill and the decode steps
 * refuse (DLA_ERR_UNSUPPORTED) until dla_cache_init resets the cache.  The
 * trace records boundaries and no merges.  Other arguments as for
 * dla_prefill; ws: at least dla_workspace_bytes(cfg, DLA_POLICY_UNBOUNDED). */
dla_status dla_unbounded_prefill(const dla_config *cfg, const void *q, const void *k,
                                 const void *v, void *o, const dla_cache *cache,
                                 const dla_trace *trace, void *ws, size_t ws_bytes,
                                 int32_t *dev_status, void *stream);

/* A ragged batch: sequence b of the call has lens[b] tokens (a device int32
 * array [B]; values are clamped to [0, T]), stored in the first lens[b]
 * rows of its [T] rows of q, k, v, as in a padded batch.  Each stream (b, h)
 * runs exactly as a call of its own with T = lens[b] would: its cache
 * advances by lens[b] tokens (lens[b] = 0 leaves it unchanged), rows
 * t >= lens[b] of o and of trace->boundary are not written, and the trace's
 * merges are its own.  The serving case the pages point to: requests of
 * different lengths prefilled in one call into their own caches.
 * `policy` is DLA_POLICY_DYNAMIC (as dla_prefill), DLA_POLICY_UNBOUNDED (as
 * dla_unbounded_prefill) or DLA_POLICY_INFO (as dla_info_policy_prefill); the
 * workspace is dla_workspace_bytes(cfg, policy) and the work is that of the
 * longest sequence per window.  Other arguments and errors as for that
 * policy's entry point. */
dla_status dla_prefill_varlen(const dla_config *cfg, int32_t policy, const int32_t *lens,
                              const void *q, const void *k, const void *v, void *o,
                              const dla_cache *cache, const dla_trace *trace, void *ws,
                              size_t ws_bytes, int32_t *dev_status, void *stream);

/* dla_decode_step for a subset of the cache's sequences (continuous
 * batching: requests that have no token this step, or have finished, stay in
 * the cache untouched).  active: device uint8 [N]; sequence n takes the step
 * when active[n] != 0.  For an inactive sequence nothing is read from q, k,
 * v and nothing is written to its cache, o, boundary or merge_i rows.  Other
 * arguments as for dla_decode_step. */
dla_status dla_decode_step_masked(const dla_cache *cache, float tau, int32_t in_dtype,
                                  const uint8_t *active, const void *q, const void *k,
                                  const void *v, void *o, uint8_t *boundary, int32_t *merge_i,
                                  void *ws, size_t ws_bytes, int32_t *dev_status, void *stream);

/* Per-stream summary of one prefill's decision trace (device arrays [B*H],
 * caller-owned; a NULL member is not written):
 *   boundaries  states the call opened (boundary flags set)
 *   merges      capacity merges of the call (the trace's merge_count)
 *   live_sum    sum over the call's tokens of the states each token read
 *               (mean live states = live_sum / T)
 *   live_max    most states a token of the call read
 *   atom_rows   sum over tiles c >= 1 of `tile` tokens of (rows of the tile) x
 *               (states live after token c * tile - 1): the states a tiled
 *               readout reads before each tile, the readout's FLOP count over
 *               2 d^2 (tile 128 for the tensor-core readout)                 */
typedef struct {
  int32_t *boundaries, *merges;
  int64_t *live_sum;
  int32_t *live_max;
  int64_t *atom_rows;
} dla_stats;

/* Reduce `trace` (as written by a prefill of T tokens for `heads` streams)
 * on `stream`, without copying it to the host: the observables the pages
 * list for a DLA memory (the Chlience page's list of what to observe:
 * boundary counts, merge frequency, live states).  The live count read by
 * token t is m_before + (boundaries at s <= t) - (merges at s <= t);
 * m_before [heads] (int32) and t_before [heads] (int64) are the streams'
 * live states and tokens seen before the call (device arrays saved from the
 * cache before it; NULL = an empty cache).  A trace whose merge_count exceeds
 * its cap sets DLA_ERR_TRACE_OVERFLOW in *dev_status (the counts then miss
 * the lost merges).  The fixed policy writes no trace. */
dla_status dla_trace_stats(const dla_trace *trace, int32_t heads, int32_t T,
                           const int32_t *m_before, const int64_t *t_before, int32_t tile,
                           const dla_stats *out, int32_t *dev_status, void *stream);

/* Workspace bytes for dla_prefill_backward with this config; 0 when the
 * config is outside its limits (d_k == d_v in {32, 64, 128}, 2 <= C <= 128,
 * T <= 4096, in_dtype DLA_F32 or DLA_BF16). */
size_t dla_backward_workspace_bytes(const dla_config *cfg);

/* Gradient of dla_prefill's output with respect to q, k and v, at the
 * decisions that prefill took (Chlience section 5.1 states, 5.2 merges, 5.3
 * readout).  The boundaries and merges are piecewise constant in the keys,
 * so wherever the forward is differentiable this is its exact gradient: the
 * decision trace is an input and is held fixed.  (The page's section 5.1 says
 * training uses a soft gate through the decisions and gives no form for it;
 * no such term is added.)
 *   cfg    the forward's config (B, H, T, d_k = d_v, C, in_dtype; tau and
 *          window unused), within dla_backward_workspace_bytes' limits;
 *   q, k, v, d_o  [B][H][T][d] in cfg->in_dtype (device): the forward's
 *          inputs and dL/do;
 *   trace  the forward's decision trace (boundary, merge_t, merge_i,
 *          merge_count, cap), from a dla_prefill that started every stream
 *          from an empty cache (merge_t then counts from 0);
 *   dq, dk, dv  [B][H][T][d] fp32 outputs (device, caller-owned);
 *   ws     device workspace of dla_backward_workspace_bytes(cfg) bytes,
 *          256-byte aligned.
 * Three kernels on `stream` (SIMT, quadratic in T).  Argument errors return
 * at once (DLA_ERR_INVALID_ARG, DLA_ERR_UNSUPPORTED, DLA_ERR_WORKSPACE); a
 * trace that does not describe such a forward (a merge off a boundary, a
 * merge index out of range, more than C live states, token 0 not a
 * boundary) sets DLA_ERR_INVALID_ARG in *dev_status, a merge_count above cap
 * DLA_ERR_TRACE_OVERFLOW, and the gradients are then unspecified. */
dla_status dla_prefill_backward(const dla_config *cfg, const void *q, const void *k, const void *v,
                                const void *d_o, const dla_trace *trace, float *dq, float *dk,
                                float *dv, void *ws, size_t ws_bytes, int32_t *dev_status,
                                void *stream);

/* Static description of a status code. */
const char *dla_status_string(dla_status status);

#ifdef __cplusplus
}
#endif

#endif /* DLA_H_ */
