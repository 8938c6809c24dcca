// dla_api.cu -- host side of the libdla C ABI: argument checks, cache and
// workspace layout, and the per-window launch sequence.
#include <string.h>

#include "dla_internal.cuh"

namespace dla {

int simt_tile_rows();
int tc_tile_rows();
bool simt_fits(int D, int C);
cudaError_t launch_trace_stats(const dla_trace &tr, int heads, int T, const int32_t *m_before,
                               const int64_t *t_before, int tile, const dla_stats &out,
                               int32_t *dev_status, cudaStream_t s);

namespace {

constexpr size_t ALIGN = 256;

size_t align_up(size_t x) { return (x + ALIGN - 1) / ALIGN * ALIGN; }

// Sequential carve-up of a device buffer (or a dry run for size queries).
struct Carver {
  char *base;
  size_t off = 0;
  template <typename T>
  T *take(size_t count) {
    T *p = base ? reinterpret_cast<T *>(base + off) : nullptr;
    off = align_up(off + count * sizeof(T));
    return p;
  }
};

bool d_ok(int32_t d) { return d == 32 || d == 64 || d == 128; }

void carve_cache(Carver &cv, dla_cache &c) {
  const size_t u = (size_t)c.N * c.H;
  c.S = cv.take<float>(u * c.C * c.d_v * c.d_k);
  c.z = cv.take<double>(u * c.C * c.d_k);
  c.n = cv.take<int64_t>(u * c.C);
  c.ts = cv.take<int64_t>(u * c.C);
  c.pair_loss = cv.take<double>(u * c.C);
  c.order = cv.take<int32_t>(u * c.C);
  c.m = cv.take<int32_t>(u);
  c.prev_k = cv.take<float>(u * c.d_k);
  c.prev_r = cv.take<double>(u);
  c.t = cv.take<int64_t>(u);
}

// The tensor-core path serves bf16 inputs with d = 128; everything else runs
// the fp32 SIMT readout.
bool use_tc(const dla_config &cfg) { return cfg.in_dtype == DLA_BF16 && cfg.d_k == 128; }

Dims make_dims(const dla_config &cfg, int policy) {
  Dims dm{};
  dm.heads = cfg.B * cfg.H;
  dm.T = cfg.T;
  const bool tc = use_tc(cfg);
  dm.M = tc ? tc_tile_rows() : simt_tile_rows();
  dm.D = cfg.d_k;
  dm.C = cfg.C;
  dm.info = policy == DLA_POLICY_INFO ? 1 : 0;
  dm.unb = policy == DLA_POLICY_UNBOUNDED ? 1 : 0;
  int W = cfg.window > 0 ? cfg.window : (tc ? 8192 : 2048);
  W = (W + dm.M - 1) / dm.M * dm.M;
  const int Tr = (cfg.T + dm.M - 1) / dm.M * dm.M;
  if (Tr > 0 && W > Tr) W = Tr;
  if (W < dm.M) W = dm.M;
  dm.W = W;
  dm.tiles = W / dm.M;
  dm.amax = dm.C;
  const int per_tile = dm.C < 2 * dm.M + 1 ? dm.C : 2 * dm.M + 1;
  // with no merges a state is frozen at most once, plus the open state at
  // every tile start
  dm.vmax = dm.unb ? dm.C + dm.tiles : dm.C + dm.tiles * per_tile;
  dm.opsmax = 4 * W + dm.tiles + 2 + dm.vmax + 8;
  dm.vbytes = dm.D * dm.D * (tc ? 2 : (int)sizeof(float));
  dm.pmax = tc ? dm.tiles * PIECES_PER_TILE : 0;
  return dm;
}

// Per-tile outputs of the tensor-core readout's prologue kernel.
void carve_pre(Carver &cv, const Dims &dm, Plan &pl) {
  if (dm.vbytes != dm.D * dm.D * 2) return;  // SIMT path: none
  const size_t g = (size_t)dm.heads * dm.tiles;
  pl.phi_q = cv.take<char>((size_t)dm.heads * dm.W * dm.D * 2);
  pl.phi_k = cv.take<char>((size_t)dm.heads * dm.W * dm.D * 2);
  pl.pre_w = cv.take<float>(g * dm.amax * dm.M);
  pl.pre_o = cv.take<char>(g * dm.M * dm.D * 2);
}

void carve_plan(Carver &cv, const Dims &dm, Plan &pl) {
  const size_t h = dm.heads;
  pl.r = cv.take<double>(h * dm.W);
  pl.b = cv.take<uint8_t>(h * dm.W);
  pl.seg_start = cv.take<int32_t>(h * (dm.W + 1));
  pl.nseg = cv.take<int32_t>(h);
  pl.z_end = cv.take<double>(h * dm.W * dm.D);
  pl.z_tile = cv.take<double>(h * dm.tiles * dm.D);
  pl.z_part = cv.take<double>(h * dm.W * dm.D);
  pl.ops = cv.take<int4>(h * dm.opsmax);
  pl.nops = cv.take<int32_t>(h);
  pl.tile_m0 = cv.take<int32_t>(h * dm.tiles);
  pl.tile_atoms = cv.take<int32_t>(h * dm.tiles * dm.amax);
  pl.tile_nev = cv.take<int32_t>(h * dm.tiles);
  pl.tile_ev_off = cv.take<int32_t>(h * dm.tiles * dm.M);
  pl.tile_ev_mrg = cv.take<int32_t>(h * dm.tiles * dm.M);
  pl.ver_z = cv.take<float>(h * dm.vmax * dm.D);
  pl.ver_n = cv.take<float>(h * dm.vmax);
  pl.ver_S = cv.take<char>(h * dm.vmax * (size_t)dm.vbytes);
  pl.slot_ver = cv.take<int32_t>(h * dm.C);
  pl.pieces = cv.take<float>(h * (size_t)dm.pmax * dm.D * dm.D);
  pl.phi_tab = cv.take<double>(4096);
  carve_pre(cv, dm, pl);
  pl.seg_info = dm.info ? cv.take<double>(h * dm.W) : nullptr;
}

// The information policy's state carried across a call's windows.
void carve_info(Carver &cv, const Dims &dm, CallArgs &ca) {
  const size_t h = dm.heads;
  ca.info_S = cv.take<double>(h * dm.D * dm.D);
  ca.info_aux = cv.take<double>(h * 4);
  ca.info_slot = cv.take<double>(h * dm.C);
}

// Fixed Fenwick policy: one pass over the call (no windows); versions are the
// nodes of a tree over whole tiles.
Dims make_dims_fenwick(const dla_config &cfg) {
  Dims dm{};
  const bool tc = use_tc(cfg);
  dm.heads = cfg.B * cfg.H;
  dm.T = cfg.T;
  dm.M = tc ? tc_tile_rows() : simt_tile_rows();
  dm.D = cfg.d_k;
  dm.C = 32;
  dm.tiles = (cfg.T + dm.M - 1) / dm.M;
  if (dm.tiles < 1) dm.tiles = 1;
  dm.W = dm.tiles * dm.M;
  dm.amax = 32;
  int nodes = 1, levels = 1;
  fen_tree_shape(cfg.T > 0 ? cfg.T : 1, dm.M, &nodes, &levels);
  dm.vmax = nodes;
  dm.opsmax = 0;
  dm.vbytes = dm.D * dm.D * (tc ? 2 : (int)sizeof(float));
  dm.fenwick = 1;
  return dm;
}

void carve_fenwick(Carver &cv, const Dims &dm, Plan &pl, float **treeS, float **treeZ) {
  const size_t h = dm.heads;
  pl.tile_m0 = cv.take<int32_t>(h * dm.tiles);
  pl.tile_atoms = cv.take<int32_t>(h * dm.tiles * dm.amax);
  pl.tile_nev = cv.take<int32_t>(h * dm.tiles);
  pl.tile_ev_off = cv.take<int32_t>(h * dm.tiles * dm.M);
  pl.tile_ev_mrg = cv.take<int32_t>(h * dm.tiles * dm.M);
  pl.ver_z = cv.take<float>(h * dm.vmax * dm.D);
  pl.ver_n = cv.take<float>(h * dm.vmax);
  pl.ver_S = cv.take<char>(h * dm.vmax * (size_t)dm.vbytes);
  *treeS = cv.take<float>(h * dm.vmax * (size_t)dm.D * dm.D);
  *treeZ = cv.take<float>(h * dm.vmax * (size_t)dm.D);
  carve_pre(cv, dm, pl);
}

bool cfg_ok(const dla_config *cfg, int policy) {
  if (!cfg) return false;
  if (cfg->B <= 0 || cfg->H <= 0 || cfg->T < 0) return false;
  if (cfg->in_dtype != DLA_F32 && cfg->in_dtype != DLA_BF16) return false;
  if (cfg->window < 0) return false;
  (void)policy;
  return true;
}

dla_status shape_ok(const dla_config *cfg, int policy) {
  if (cfg->d_k != cfg->d_v || !d_ok(cfg->d_k)) return DLA_ERR_UNSUPPORTED;
  if ((policy == DLA_POLICY_DYNAMIC || policy == DLA_POLICY_INFO) && (cfg->C < 2 || cfg->C > 128))
    return DLA_ERR_UNSUPPORTED;
  if (policy == DLA_POLICY_UNBOUNDED) {
    if (cfg->C < 2 || cfg->C > DLA_MAX_SLOTS) return DLA_ERR_UNSUPPORTED;
    // the SIMT readout keeps every atom's logits of a tile in shared memory
    if (!use_tc(*cfg) && !simt_fits(cfg->d_k, cfg->C)) return DLA_ERR_UNSUPPORTED;
  }
  return DLA_OK;
}

// The auxiliary streams of a prefill call and their fork / join events, one
// set per host thread and device, created on first use and kept for the
// thread's lifetime (non-blocking, so they never synchronise with the legacy
// stream).  `s` runs the score and sums at normal priority; `se` runs the
// engine at the highest priority: it is latency-bound and on the critical
// path of a single window, so its few CTAs should get SMs first.  With the
// tensor-core readout, `sb` runs the state builder, `sx` the materializer at
// the highest priority and `sp` the phi operands and the readout's prologue
// beside it at the lowest, so that the materializer's CTAs are placed first.
// Windows cycle through NPLAN plans: a plan is reused three windows later, so
// window w + 1's decisions and window w + 2's never wait for window w's
// readout.
constexpr int NPLAN = 3;
enum { EV_START = 0, EV_SCAN, EV_SUMS, EV_ENGINE, EV_BUILD, EV_MAT, EV_PRE, EV_DONE0,
       EV_COUNT = EV_DONE0 + NPLAN };
int plan_count(const dla_config &cfg, const Dims &dm) {
  const int windows = (cfg.T + dm.W - 1) / dm.W;
  return windows < 1 ? 1 : (windows < NPLAN ? windows : NPLAN);
}
struct Aux {
  cudaStream_t s = nullptr, se = nullptr, sp = nullptr, sx = nullptr, sb = nullptr;
  cudaEvent_t ev[EV_COUNT] = {};
  bool ok = false;
};
constexpr int MAX_DEVICES = 64;

Aux *aux_streams() {
  thread_local Aux aux[MAX_DEVICES];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= MAX_DEVICES) return nullptr;
  Aux &a = aux[dev];
  if (!a.ok) {
    int lo = 0, hi = 0;
    if (cudaDeviceGetStreamPriorityRange(&lo, &hi) != cudaSuccess) return nullptr;
    if (!a.s && cudaStreamCreateWithFlags(&a.s, cudaStreamNonBlocking) != cudaSuccess) return nullptr;
    if (!a.se && cudaStreamCreateWithPriority(&a.se, cudaStreamNonBlocking, hi) != cudaSuccess)
      return nullptr;
    if (!a.sp && cudaStreamCreateWithPriority(&a.sp, cudaStreamNonBlocking, lo) != cudaSuccess)
      return nullptr;
    if (!a.sx && cudaStreamCreateWithPriority(&a.sx, cudaStreamNonBlocking, hi) != cudaSuccess)
      return nullptr;
    if (!a.sb && cudaStreamCreateWithFlags(&a.sb, cudaStreamNonBlocking) != cudaSuccess) return nullptr;
    for (cudaEvent_t &e : a.ev)
      if (!e && cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return nullptr;
    a.ok = true;
  }
  return &a;
}

}  // namespace
}  // namespace dla

using namespace dla;

extern "C" {

const char *dla_status_string(dla_status s) {
  switch (s) {
    case DLA_OK: return "ok";
    case DLA_ERR_INVALID_ARG: return "invalid argument";
    case DLA_ERR_UNSUPPORTED:
      return "unsupported shape (need d_k == d_v in {32, 64, 128}, 2 <= C <= 128) or a cache "
             "this policy cannot continue";
    case DLA_ERR_CUDA: return "CUDA launch failed";
    case DLA_ERR_TRACE_OVERFLOW: return "more merges than the trace capacity";
    case DLA_ERR_WORKSPACE: return "workspace smaller than dla_workspace_bytes()";
    case DLA_ERR_INVARIANT: return "device invariant violated";
    case DLA_ERR_TIMEOUT: return "a bounded device wait timed out";
    case DLA_ERR_CAPACITY: return "the unbounded policy needs more states than the cache has slots";
  }
  return "unknown status";
}

size_t dla_cache_bytes(int32_t N, int32_t H, int32_t C, int32_t d_k, int32_t d_v) {
  if (N <= 0 || H <= 0 || C <= 0 || d_k <= 0 || d_v <= 0) return 0;
  dla_cache c{};
  c.N = N;
  c.H = H;
  c.C = C;
  c.d_k = d_k;
  c.d_v = d_v;
  Carver cv{nullptr};
  carve_cache(cv, c);
  return cv.off;
}

dla_status dla_cache_init(dla_cache *cache, int32_t N, int32_t H, int32_t C, int32_t d_k,
                          int32_t d_v, void *dev_base, size_t bytes, void *stream) {
  if (!cache || !dev_base) return DLA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(dev_base) % ALIGN != 0) return DLA_ERR_INVALID_ARG;
  const size_t need = dla_cache_bytes(N, H, C, d_k, d_v);
  if (need == 0) return DLA_ERR_INVALID_ARG;
  if (bytes < need) return DLA_ERR_WORKSPACE;
  if (d_k != d_v || !d_ok(d_k) || C < 2 || C > DLA_MAX_SLOTS) return DLA_ERR_UNSUPPORTED;
  dla_cache c{};
  c.N = N;
  c.H = H;
  c.C = C;
  c.d_k = d_k;
  c.d_v = d_v;
  Carver cv{static_cast<char *>(dev_base)};
  carve_cache(cv, c);
  // S is carved first; everything after it is reset
  const size_t s_end = reinterpret_cast<char *>(c.z) - static_cast<char *>(dev_base);
  if (cudaMemsetAsync(static_cast<char *>(dev_base) + s_end, 0, need - s_end,
                      static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return DLA_ERR_CUDA;
  *cache = c;
  return DLA_OK;
}

size_t dla_workspace_bytes(const dla_config *cfg, int32_t policy) {
  if (!cfg_ok(cfg, policy) || shape_ok(cfg, policy) != DLA_OK) return 0;
  if (policy == DLA_POLICY_FENWICK) {
    const Dims dm = make_dims_fenwick(*cfg);
    Plan pl{};
    float *a, *b;
    Carver cv{nullptr};
    carve_fenwick(cv, dm, pl, &a, &b);
    return cv.off;
  }
  if (policy != DLA_POLICY_DYNAMIC && policy != DLA_POLICY_INFO && policy != DLA_POLICY_UNBOUNDED)
    return 0;
  const Dims dm = make_dims(*cfg, policy);
  Plan pl{};
  Carver cv{nullptr};
  for (int i = 0, n = plan_count(*cfg, dm); i < n; i++) carve_plan(cv, dm, pl);
  if (policy == DLA_POLICY_INFO) {
    CallArgs ca{};
    carve_info(cv, dm, ca);
  }
  return cv.off;
}

}  // extern "C"

namespace {

// A prefill call of the dynamic policy (cosine score, Ward merges) or the
// information policy (state score, density merges): the same windows,
// streams and kernels but the score and the engine's pair criterion.
dla_status prefill_impl(int policy, const dla_config *cfg, const void *q, const void *k,
                        const void *v, void *o, const dla_cache *cache, const dla_trace *trace,
                        void *ws, size_t ws_bytes, int32_t *dev_status, void *stream,
                        const int32_t *lens = nullptr) {
  if (!cfg_ok(cfg, policy) || !cache) return DLA_ERR_INVALID_ARG;
  const dla_status sh = shape_ok(cfg, policy);
  if (sh != DLA_OK) return sh;
  if (cache->N != cfg->B || cache->H != cfg->H || cache->C != cfg->C || cache->d_k != cfg->d_k ||
      cache->d_v != cfg->d_v)
    return DLA_ERR_INVALID_ARG;
  if (cfg->T == 0) return DLA_OK;
  if (!q || !k || !v || !o || !ws) return DLA_ERR_INVALID_ARG;
  if (trace && (!trace->boundary || !trace->merge_t || !trace->merge_i || !trace->merge_count ||
                trace->cap < 0))
    return DLA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(ws) % ALIGN != 0) return DLA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(q) % 16 || reinterpret_cast<uintptr_t>(k) % 16 ||
      reinterpret_cast<uintptr_t>(v) % 16 || reinterpret_cast<uintptr_t>(o) % 16)
    return DLA_ERR_INVALID_ARG;
  const bool info = policy == DLA_POLICY_INFO;
  const Dims dm = make_dims(*cfg, policy);
  Plan plans[NPLAN] = {};
  Carver cv{static_cast<char *>(ws)};
  const int nplan = plan_count(*cfg, dm);
  for (int i = 0; i < nplan; i++) carve_plan(cv, dm, plans[i]);
  CallArgs ca{};
  if (info) carve_info(cv, dm, ca);
  if (cv.off > ws_bytes) return DLA_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  Aux *ax = aux_streams();
  if (!ax) return DLA_ERR_CUDA;
  cudaStream_t sd = ax->s;   // decisions: score, pieces, sums
  cudaStream_t se = ax->se;  // the engine
  cudaStream_t sp = ax->sp;  // the tensor-core readout's prologue
  cudaStream_t sx = ax->sx;  // the materializer, with the tensor-core readout
  cudaStream_t sb = ax->sb;  // the tensor-core state builder
  ca.q = q;
  ca.k = k;
  ca.v = v;
  ca.o = o;
  ca.in_dtype = cfg->in_dtype;
  ca.tau = cfg->tau;
  ca.cache = *cache;
  ca.lens = lens;
  ca.H = cfg->H;
  if (trace) {
    ca.trace = *trace;
    if (cudaMemsetAsync(trace->merge_count, 0, sizeof(int32_t) * dm.heads, s) != cudaSuccess)
      return DLA_ERR_CUDA;
  } else {
    memset(&ca.trace, 0, sizeof ca.trace);
  }
  if (info && cudaMemsetAsync(ca.info_slot, 0, sizeof(double) * dm.heads * dm.C, s) != cudaSuccess)
    return DLA_ERR_CUDA;
  ca.dev_status = dev_status;
  // Fork: the decision kernels and the engine run on the auxiliary stream,
  // the state build, materializer and readout on the caller's stream.  The
  // builder needs only the boundary flags, so it overlaps the engine; window
  // w + 1's decisions overlap window w's heavy kernels.  Every
  // auxiliary launch is ordered before a later wait of the caller's stream,
  // so the call ends (joins) on the caller's stream.
  if (cudaEventRecord(ax->ev[EV_START], s) != cudaSuccess ||
      cudaStreamWaitEvent(sd, ax->ev[EV_START], 0) != cudaSuccess ||
      cudaStreamWaitEvent(sp, ax->ev[EV_START], 0) != cudaSuccess)
    return DLA_ERR_CUDA;
  const bool tc = use_tc(*cfg);
  dla_profile *pf = cfg->profile;
  int wi = 0;
  for (int w0 = 0; w0 < cfg->T; w0 += dm.W, wi++) {
    const int pi = wi % nplan;  // this window's plan, last used by window wi - nplan
    const Plan &pl = plans[pi];
    const bool reuse = wi >= nplan;
    ca.w0 = w0;
    ca.Tw = cfg->T - w0 < dm.W ? cfg->T - w0 : dm.W;
    cudaError_t e = cudaSuccess;
    // this plan was last read by window wi - nplan's readout.  The score and scan
    // of a later window read only the call's input; the piece sums read the
    // cache's open state, written by window wi - 1's engine
    if (reuse && cudaStreamWaitEvent(sd, ax->ev[EV_DONE0 + pi], 0) != cudaSuccess)
      return DLA_ERR_CUDA;
    if (info) {
      ProfScope ps(pf, DLA_K_INFO_SCORE, sd);
      e = launch_info_score(dm, pl, ca, sd);
    } else {
      ProfScope ps(pf, DLA_K_SCORE, sd);
      e = launch_score(dm, pl, ca, DLA_POLICY_DYNAMIC, sd);
    }
    if (e != cudaSuccess) return DLA_ERR_CUDA;
    { ProfScope ps(pf, DLA_K_SEGSCAN, sd); e = launch_segscan(dm, pl, ca, sd); }
    if (e != cudaSuccess || cudaEventRecord(ax->ev[EV_SCAN], sd) != cudaSuccess) return DLA_ERR_CUDA;
    if (wi >= 1 && cudaStreamWaitEvent(sd, ax->ev[EV_ENGINE], 0) != cudaSuccess)
      return DLA_ERR_CUDA;
    { ProfScope ps(pf, DLA_K_SEGSUM, sd); e = launch_segsum(dm, pl, ca, sd); }
    if (e != cudaSuccess || cudaEventRecord(ax->ev[EV_SUMS], sd) != cudaSuccess ||
        cudaStreamWaitEvent(se, ax->ev[EV_SUMS], 0) != cudaSuccess)
      return DLA_ERR_CUDA;
    { ProfScope ps(pf, DLA_K_ENGINE, se); e = launch_engine(dm, pl, ca, se); }
    if (e != cudaSuccess || cudaEventRecord(ax->ev[EV_ENGINE], se) != cudaSuccess) return DLA_ERR_CUDA;
    if (tc) {
      // phi(q) of the window beside the latency-bound engine (after the
      // score, whose memory traffic it would slow); the plan's phi buffers
      // were last read by window wi - nplan's readout
      if (cudaStreamWaitEvent(sp, ax->ev[EV_SCAN], 0) != cudaSuccess) return DLA_ERR_CUDA;
      if (reuse && cudaStreamWaitEvent(sp, ax->ev[EV_DONE0 + pi], 0) != cudaSuccess)
        return DLA_ERR_CUDA;
      { ProfScope ps(pf, DLA_K_PHI, sp); e = launch_phi_tc(dm, pl, ca, sp); }
      if (e != cudaSuccess) return DLA_ERR_CUDA;
    }
    if (tc) {
      // the builder reads only the boundary flags (after the score, so it does
      // not slow it); it overlaps the engine and the previous window's
      // readout.  Its pieces were last read by window wi - nplan's materializer,
      // before the decision stream's wait above
      if (cudaStreamWaitEvent(sb, ax->ev[EV_SCAN], 0) != cudaSuccess) return DLA_ERR_CUDA;
      { ProfScope ps(pf, DLA_K_BUILD, sb); e = launch_build_tc(dm, pl, ca, sb); }
      if (e != cudaSuccess || cudaEventRecord(ax->ev[EV_BUILD], sb) != cudaSuccess) return DLA_ERR_CUDA;
    }
    if (tc) {
      // the readout's prologue needs the engine's atom lists and means, not
      // the versions: it runs beside the materializer
      if (cudaStreamWaitEvent(sp, ax->ev[EV_ENGINE], 0) != cudaSuccess ||
          cudaStreamWaitEvent(sp, ax->ev[EV_BUILD], 0) != cudaSuccess)  // phi(k) tiles
        return DLA_ERR_CUDA;
      { ProfScope ps(pf, DLA_K_READOUT_PRE, sp); e = launch_readout_pre_tc(dm, pl, ca, sp); }
      if (e != cudaSuccess || cudaEventRecord(ax->ev[EV_PRE], sp) != cudaSuccess) return DLA_ERR_CUDA;
    }
    // the materializer: after the engine (ops) and the builder (pieces); on
    // sx it also waits for window wi - nplan's readout, the last reader of this
    // plan's versions, and for the previous materializer through stream order
    cudaStream_t sm_ = tc ? sx : s;
    if (cudaStreamWaitEvent(sm_, ax->ev[EV_ENGINE], 0) != cudaSuccess) return DLA_ERR_CUDA;
    if (tc && (cudaStreamWaitEvent(sx, ax->ev[EV_BUILD], 0) != cudaSuccess ||
               (reuse && cudaStreamWaitEvent(sx, ax->ev[EV_DONE0 + pi], 0) != cudaSuccess)))
      return DLA_ERR_CUDA;
    { ProfScope ps(pf, DLA_K_MATERIALIZE, sm_); e = launch_materialize(dm, pl, ca, sm_, tc); }
    if (e != cudaSuccess) return DLA_ERR_CUDA;
    if (tc && (cudaEventRecord(ax->ev[EV_MAT], sx) != cudaSuccess ||
               cudaStreamWaitEvent(s, ax->ev[EV_MAT], 0) != cudaSuccess ||
               cudaStreamWaitEvent(s, ax->ev[EV_PRE], 0) != cudaSuccess))
      return DLA_ERR_CUDA;
    {
      ProfScope ps(pf, DLA_K_READOUT, s);
      e = tc ? launch_readout_tc(dm, pl, ca, s) : launch_readout_simt(dm, pl, ca, s);
    }
    if (e != cudaSuccess || cudaEventRecord(ax->ev[EV_DONE0 + pi], s) != cudaSuccess)
      return DLA_ERR_CUDA;
  }
  return DLA_OK;
}

dla_status decode_impl(const dla_cache *cache, float tau, int32_t in_dtype, const uint8_t *active,
                       const void *q, const void *k, const void *v, void *o, uint8_t *boundary,
                       int32_t *merge_i, void *ws, size_t ws_bytes, int32_t *dev_status,
                       void *stream, dla_profile *profile) {
  if (!cache || !q || !k || !v || !o || !ws) return DLA_ERR_INVALID_ARG;
  if (in_dtype != DLA_F32 && in_dtype != DLA_BF16) return DLA_ERR_INVALID_ARG;
  if (!cache->S || !cache->z || !cache->order || !cache->m) return DLA_ERR_INVALID_ARG;
  const size_t need = dla_decode_workspace_bytes(cache->N, cache->H, cache->C, cache->d_k,
                                                 cache->d_v);
  if (need == 0) return DLA_ERR_UNSUPPORTED;
  if (ws_bytes < need) return DLA_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(ws) % ALIGN != 0) return DLA_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  {
    ProfScope ps(profile, DLA_K_DECODE_DECIDE, s);
    e = launch_decode_decide(*cache, tau, in_dtype, q, k, ws, boundary, merge_i, dev_status, s,
                             active);
  }
  if (e != cudaSuccess) return DLA_ERR_CUDA;
  {
    ProfScope ps(profile, DLA_K_DECODE_STREAM, s);
    e = launch_decode_stream(*cache, in_dtype, q, k, v, o, ws, s);
  }
  if (e != cudaSuccess) return DLA_ERR_CUDA;
  return DLA_OK;
}

}  // namespace

extern "C" {

dla_status dla_prefill(const dla_config *cfg, const void *q, const void *k, const void *v,
                       void *o, const dla_cache *cache, const dla_trace *trace, void *ws,
                       size_t ws_bytes, int32_t *dev_status, void *stream) {
  return prefill_impl(DLA_POLICY_DYNAMIC, cfg, q, k, v, o, cache, trace, ws, ws_bytes,
                      dev_status, stream);
}

dla_status dla_info_policy_prefill(const dla_config *cfg, const void *q, const void *k,
                                   const void *v, void *o, const dla_cache *cache,
                                   const dla_trace *trace, void *ws, size_t ws_bytes,
                                   int32_t *dev_status, void *stream) {
  return prefill_impl(DLA_POLICY_INFO, cfg, q, k, v, o, cache, trace, ws, ws_bytes, dev_status,
                      stream);
}

dla_status dla_unbounded_prefill(const dla_config *cfg, const void *q, const void *k,
                                 const void *v, void *o, const dla_cache *cache,
                                 const dla_trace *trace, void *ws, size_t ws_bytes,
                                 int32_t *dev_status, void *stream) {
  return prefill_impl(DLA_POLICY_UNBOUNDED, cfg, q, k, v, o, cache, trace, ws, ws_bytes,
                      dev_status, stream);
}

dla_status dla_prefill_varlen(const dla_config *cfg, int32_t policy, const int32_t *lens,
                              const void *q, const void *k, const void *v, void *o,
                              const dla_cache *cache, const dla_trace *trace, void *ws,
                              size_t ws_bytes, int32_t *dev_status, void *stream) {
  if (!lens) return DLA_ERR_INVALID_ARG;
  if (policy != DLA_POLICY_DYNAMIC && policy != DLA_POLICY_INFO && policy != DLA_POLICY_UNBOUNDED)
    return DLA_ERR_INVALID_ARG;
  return prefill_impl(policy, cfg, q, k, v, o, cache, trace, ws, ws_bytes, dev_status, stream,
                      lens);
}

dla_status dla_trace_stats(const dla_trace *trace, int32_t heads, int32_t T,
                           const int32_t *m_before, const int64_t *t_before, int32_t tile,
                           const dla_stats *out, int32_t *dev_status, void *stream) {
  if (!trace || !out || heads <= 0 || T < 0 || tile < 0) return DLA_ERR_INVALID_ARG;
  if (!trace->boundary || !trace->merge_count || (trace->cap > 0 && !trace->merge_t) ||
      trace->cap < 0)
    return DLA_ERR_INVALID_ARG;
  if (T == 0) return DLA_OK;
  if (launch_trace_stats(*trace, heads, T, m_before, t_before, tile, *out, dev_status,
                         static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return DLA_ERR_CUDA;
  return DLA_OK;
}

size_t dla_decode_workspace_bytes(int32_t N, int32_t H, int32_t C, int32_t d_k, int32_t d_v) {
  if (N <= 0 || H <= 0 || C < 2 || C > 128 || d_k != d_v || !d_ok(d_k)) return 0;
  return decode_ws_bytes(N, H, C);
}

dla_status dla_decode_step_masked(const dla_cache *cache, float tau, int32_t in_dtype,
                                  const uint8_t *active, const void *q, const void *k,
                                  const void *v, void *o, uint8_t *boundary, int32_t *merge_i,
                                  void *ws, size_t ws_bytes, int32_t *dev_status, void *stream) {
  if (!active) return DLA_ERR_INVALID_ARG;
  return decode_impl(cache, tau, in_dtype, active, q, k, v, o, boundary, merge_i, ws, ws_bytes,
                     dev_status, stream, nullptr);
}

dla_status dla_decode_step(const dla_cache *cache, float tau, int32_t in_dtype, const void *q,
                           const void *k, const void *v, void *o, uint8_t *boundary,
                           int32_t *merge_i, void *ws, size_t ws_bytes, int32_t *dev_status,
                           void *stream, dla_profile *profile) {
  return decode_impl(cache, tau, in_dtype, nullptr, q, k, v, o, boundary, merge_i, ws, ws_bytes,
                     dev_status, stream, profile);
}


dla_status dla_decode_step_static(const dla_cache *cache, float tau, int32_t in_dtype,
                                  const void *q, const void *k, const void *v, void *o,
                                  uint8_t *boundary, int32_t *merge_i, int32_t *dev_status,
                                  void *stream) {
  if (!cache || !q || !k || !v || !o) return DLA_ERR_INVALID_ARG;
  if (in_dtype != DLA_F32 && in_dtype != DLA_BF16) return DLA_ERR_INVALID_ARG;
  if (!cache->S || !cache->z || !cache->order || !cache->m) return DLA_ERR_INVALID_ARG;
  const size_t need = dla_decode_workspace_bytes(cache->N, cache->H, cache->C, cache->d_k,
                                                 cache->d_v);
  if (need == 0) return DLA_ERR_UNSUPPORTED;
  if (need > static_decode_max_bytes()) return DLA_ERR_WORKSPACE;
  void *ws = nullptr;
  if (static_decode_scratch(&ws) != cudaSuccess) return DLA_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (launch_decode_decide(*cache, tau, in_dtype, q, k, ws, boundary, merge_i, dev_status, s) !=
      cudaSuccess)
    return DLA_ERR_CUDA;
  if (launch_decode_stream(*cache, in_dtype, q, k, v, o, ws, s) != cudaSuccess) return DLA_ERR_CUDA;
  return DLA_OK;
}

dla_status dla_fixed_policy_prefill(const dla_config *cfg, const void *q, const void *k,
                                    const void *v, void *o, void *ws, size_t ws_bytes,
                                    int32_t *dev_status, void *stream) {
  if (!cfg_ok(cfg, DLA_POLICY_FENWICK)) return DLA_ERR_INVALID_ARG;
  const dla_status sh = shape_ok(cfg, DLA_POLICY_FENWICK);
  if (sh != DLA_OK) return sh;
  if (cfg->T == 0) return DLA_OK;
  if (!q || !k || !v || !o || !ws) return DLA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(ws) % ALIGN != 0) return DLA_ERR_INVALID_ARG;
  const bool tc = use_tc(*cfg);
  if (tc && (reinterpret_cast<uintptr_t>(q) % 16 || reinterpret_cast<uintptr_t>(k) % 16 ||
             reinterpret_cast<uintptr_t>(v) % 16 || reinterpret_cast<uintptr_t>(o) % 16))
    return DLA_ERR_INVALID_ARG;
  const Dims dm = make_dims_fenwick(*cfg);
  Plan pl{};
  float *treeS = nullptr, *treeZ = nullptr;
  Carver cv{static_cast<char *>(ws)};
  carve_fenwick(cv, dm, pl, &treeS, &treeZ);
  if (cv.off > ws_bytes) return DLA_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  CallArgs ca{};
  ca.q = q;
  ca.k = k;
  ca.v = v;
  ca.o = o;
  ca.in_dtype = cfg->in_dtype;
  ca.tau = cfg->tau;
  ca.w0 = 0;
  ca.Tw = cfg->T;
  ca.dev_status = dev_status;
  memset(&ca.trace, 0, sizeof ca.trace);
  dla_profile *pf = cfg->profile;
  cudaError_t e;
  Aux *ax = tc ? aux_streams() : nullptr;
  if (tc && !ax) return DLA_ERR_CUDA;
  if (tc) {
    // phi(q) needs only the input: beside the tree build (the leaves store
    // the phi(k) tiles)
    cudaStream_t sp = ax->sp;
    if (cudaEventRecord(ax->ev[EV_START], s) != cudaSuccess ||
        cudaStreamWaitEvent(sp, ax->ev[EV_START], 0) != cudaSuccess)
      return DLA_ERR_CUDA;
    { ProfScope ps(pf, DLA_K_PHI, sp); e = launch_phi_tc(dm, pl, ca, sp); }
    if (e != cudaSuccess || cudaEventRecord(ax->ev[EV_PRE], sp) != cudaSuccess) return DLA_ERR_CUDA;
  }
  { ProfScope ps(pf, DLA_K_ENGINE, s); e = launch_fenwick(dm, pl, ca, treeS, treeZ, tc, false, s); }
  if (e != cudaSuccess) return DLA_ERR_CUDA;
  if (tc) {
    // the prologue needs the plan and the nodes' means, not their states: it
    // runs beside the tree levels
    cudaStream_t sp = ax->sp;
    if (cudaEventRecord(ax->ev[EV_SUMS], s) != cudaSuccess ||
        cudaStreamWaitEvent(sp, ax->ev[EV_SUMS], 0) != cudaSuccess)
      return DLA_ERR_CUDA;
    { ProfScope ps(pf, DLA_K_READOUT_PRE, sp); e = launch_readout_pre_tc(dm, pl, ca, sp); }
    if (e != cudaSuccess || cudaEventRecord(ax->ev[EV_PRE], sp) != cudaSuccess) return DLA_ERR_CUDA;
  }
  { ProfScope ps(pf, DLA_K_MATERIALIZE, s); e = launch_fenwick(dm, pl, ca, treeS, treeZ, tc, true, s); }
  if (e != cudaSuccess) return DLA_ERR_CUDA;
  if (tc && cudaStreamWaitEvent(s, ax->ev[EV_PRE], 0) != cudaSuccess) return DLA_ERR_CUDA;
  {
    ProfScope ps(pf, DLA_K_READOUT, s);
    e = tc ? launch_readout_tc(dm, pl, ca, s) : launch_readout_simt(dm, pl, ca, s);
  }
  if (e != cudaSuccess) return DLA_ERR_CUDA;
  return DLA_OK;
}

}  // extern "C"
