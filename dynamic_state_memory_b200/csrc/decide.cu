// decide.cu -- decision kernels of a DLA prefill window.
//
//   k_score    r_t = 1 - cos(k_t, k_{t-1}) in fp64 and the boundary flag
//              b_t = not (r_t < tau and r_{t-1} < tau), one thread per token
//              (ai-feeds.com "Dynamic Linear Attention" summary, section
//              信息感知的动态状态合并: a token joins only when it and its
//              predecessor are low-information; Chlience section 5.1: b_t = 1
//              opens a new state).
//   k_segscan  window pieces: {0} and every boundary t > 0 (warp ballots).
//   k_segsum   z = sum of phi(k) per piece in fp64, token by token, and the open
//              state's partial z before each readout tile.
//   k_engine   one warp per head walks tiles and boundaries in time order:
//              seals, capacity merges by least Ward loss (Chlience section 5.2
//              and Corollary 1), slot allocation; emits the materializer op
//              list, the per-tile atoms/events and the merge trace.
//
// Arithmetic that decides an integer is fp64 with explicit round-to-nearest
// intrinsics (no contraction): r_t is summed in index order exactly like the
// CPU oracle, so boundaries are bit-identical; Ward losses use a fixed warp
// tree order, so merge choices agree whenever the best and second-best losses
// differ by more than rounding.
#include "dla_internal.cuh"

namespace dla {
namespace {

constexpr unsigned FULL = 0xffffffffu;

__device__ double score_fp64(const void *k, int32_t dt, size_t a, size_t b, const float *bprev,
                             int D) {
  // a: row of k_t; b: row of k_{t-1} in k (ignored when bprev != nullptr)
  double dot = 0.0, na = 0.0, nb = 0.0;
  for (int c = 0; c < D; c++) {
    double x = (double)load_in(k, dt, a + c);
    double y = bprev ? (double)bprev[c] : (double)load_in(k, dt, b + c);
    dot = __dadd_rn(dot, __dmul_rn(x, y));
  }
  for (int c = 0; c < D; c++) {
    double x = (double)load_in(k, dt, a + c);
    na = __dadd_rn(na, __dmul_rn(x, x));
  }
  for (int c = 0; c < D; c++) {
    double y = bprev ? (double)bprev[c] : (double)load_in(k, dt, b + c);
    nb = __dadd_rn(nb, __dmul_rn(y, y));
  }
  if (na == 0.0 || nb == 0.0) return 1.0;
  return __dsub_rn(1.0, __ddiv_rn(dot, __dmul_rn(__dsqrt_rn(na), __dsqrt_rn(nb))));
}

// r for window-local token tl of head u (global index tg = t0 + tl).
__device__ double score_at(const Dims &dm, const CallArgs &ca, int u, int tl, int64_t t0) {
  if (t0 + tl == 0) return 0.0;
  const int D = dm.D;
  size_t row = ((size_t)u * dm.T + ca.w0 + tl) * D;
  if (tl == 0) return score_fp64(ca.k, ca.in_dtype, row, 0, ca.cache.prev_k + (size_t)u * D, D);
  return score_fp64(ca.k, ca.in_dtype, row, row - D, nullptr, D);
}

__global__ void k_score(Dims dm, Plan pl, CallArgs ca, int policy) {
  const int u = blockIdx.y;
  const int tl = blockIdx.x * blockDim.x + threadIdx.x;
  __shared__ double rprev[1];
  const int64_t t0 = ca.cache.t[u];
  double r = 0.0;
  if (policy == DLA_POLICY_DYNAMIC) {
    if (threadIdx.x == 0) {
      const int tp = blockIdx.x * blockDim.x - 1;  // token before this block
      rprev[0] = tp < 0 ? ca.cache.prev_r[u] : score_at(dm, ca, u, tp, t0);
    }
    if (tl < ca.Tw) r = score_at(dm, ca, u, tl, t0);
  }
  __shared__ double rs[256];
  rs[threadIdx.x] = r;
  __syncthreads();
  if (tl >= ca.Tw) return;
  uint8_t b = 1;
  if (policy == DLA_POLICY_DYNAMIC) {
    const double rp = threadIdx.x == 0 ? rprev[0] : rs[threadIdx.x - 1];
    const double tau = (double)ca.tau;
    const bool join = (t0 + tl > 0) && (r < tau) && (rp < tau);
    b = join ? 0 : 1;
  }
  pl.r[(size_t)u * dm.W + tl] = r;
  pl.b[(size_t)u * dm.W + tl] = b;
  if (ca.trace.boundary) ca.trace.boundary[(size_t)u * dm.T + ca.w0 + tl] = b;
}

// Pieces of the window: seg_start = {0} and every t > 0 with b_t = 1.
__global__ void k_segscan(Dims dm, Plan pl, CallArgs ca) {
  const int u = blockIdx.x;
  const uint8_t *b = pl.b + (size_t)u * dm.W;
  int32_t *ss = pl.seg_start + (size_t)u * (dm.W + 1);
  __shared__ int warp_tot[32];
  __shared__ int base;
  if (threadIdx.x == 0) {
    base = 1;
    ss[0] = 0;
  }
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  for (int c0 = 0; c0 < ca.Tw; c0 += blockDim.x) {
    const int t = c0 + threadIdx.x;
    const bool f = t > 0 && t < ca.Tw && b[t];
    const unsigned bal = __ballot_sync(FULL, f);
    if (lane == 0) warp_tot[warp] = __popc(bal);
    __syncthreads();
    int off = 0;
    for (int w = 0; w < warp; w++) off += warp_tot[w];
    if (f) ss[base + off + __popc(bal & ((1u << lane) - 1u))] = t;
    __syncthreads();
    if (threadIdx.x == 0) {
      int tot = 0;
      for (int w = 0; w < nw; w++) tot += warp_tot[w];
      base += tot;
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) pl.nseg[u] = base;
}

// z per piece (fp64, token order) and the open state's z before each tile.
__global__ void k_segsum(Dims dm, Plan pl, CallArgs ca) {
  const int u = blockIdx.y;
  const int c = threadIdx.x;  // dimension
  const int D = dm.D;
  const int nseg = pl.nseg[u];
  const int32_t *ss = pl.seg_start + (size_t)u * (dm.W + 1);
  const uint8_t *b = pl.b + (size_t)u * dm.W;
  for (int j = blockIdx.x; j < nseg; j += gridDim.x) {
    const int s0 = ss[j];
    const int s1 = j + 1 < nseg ? ss[j + 1] : ca.Tw;
    double z = 0.0;
    if (j == 0 && b[0] == 0) {
      // continuation of the cache's open state: keep summing its z in order
      const int m = ca.cache.m[u];
      const int os = ca.cache.order[(size_t)u * dm.C + m - 1];
      z = ca.cache.z[((size_t)u * dm.C + os) * D + c];
    }
    for (int s = s0; s < s1; s++) {
      const double x = (double)load_in(ca.k, ca.in_dtype, ((size_t)u * dm.T + ca.w0 + s) * D + c);
      z = __dadd_rn(z, phi64(x));
      if ((s + 1) % dm.M == 0 && (s + 1) < ca.Tw)
        pl.z_tile[((size_t)u * dm.tiles + (s + 1) / dm.M) * D + c] = z;
    }
    pl.z_end[((size_t)u * dm.W + j) * D + c] = z;
  }
}

// ---------------------------------------------------------------- engine ----

struct Eng {
  const Dims *dm;
  const Plan *pl;
  const CallArgs *ca;
  int u, lane, C, D;
  int32_t *order;
  int64_t *n, *ts;
  double *z, *loss;
  int32_t *slot_ver;
  int4 *ops;
  int nops, nver, m;
  uint32_t used[4];

  __device__ void emit(int op, int a, int b, int c) {
    if (nops < dm->opsmax) {
      if (lane == 0) ops[nops] = make_int4(op, a, b, c);
    } else if (lane == 0) {
      set_status(ca->dev_status, DLA_ERR_INVARIANT);
    }
    nops++;
  }
  __device__ double ward(int sa, int sb) const {
    const double na = (double)n[sa], nb = (double)n[sb];
    const double *za = z + (size_t)sa * D, *zb = z + (size_t)sb * D;
    double s = 0.0;
    for (int c = lane; c < D; c += 32) {
      const double diff = __dsub_rn(__ddiv_rn(za[c], na), __ddiv_rn(zb[c], nb));
      s = __dadd_rn(s, __dmul_rn(diff, diff));
    }
    for (int off = 16; off; off >>= 1) s = __dadd_rn(s, __shfl_down_sync(FULL, s, off));
    s = __shfl_sync(FULL, s, 0);
    const double f = __ddiv_rn(__dmul_rn(na, nb), __dadd_rn(na, nb));
    return __dmul_rn(f, s);
  }
  __device__ int alloc_slot() {
    for (int w = 0; w < 4; w++) {
      const uint32_t freeb = ~used[w];
      if (w * 32 < C && freeb) {
        const int bit = __ffs(freeb) - 1;
        const int slot = w * 32 + bit;
        if (slot < C) {
          used[w] |= 1u << bit;
          return slot;
        }
      }
    }
    if (lane == 0) set_status(ca->dev_status, DLA_ERR_INVARIANT);
    return 0;
  }
  __device__ void free_slot(int s) { used[s >> 5] &= ~(1u << (s & 31)); }
  // New version of `slot` with mean phi(k) = zsrc / cnt.
  __device__ int new_version(int slot, const double *zsrc, int64_t cnt) {
    const int v = nver++;
    if (v >= dm->vmax) {
      if (lane == 0) set_status(ca->dev_status, DLA_ERR_INVARIANT);
      return dm->vmax - 1;
    }
    emit(OP_SHADOW, slot, v, 0);
    float *mu = pl->ver_mu + ((size_t)u * dm->vmax + v) * D;
    const double dn = (double)cnt;
    for (int c = lane; c < D; c += 32) mu[c] = (float)__ddiv_rn(zsrc[c], dn);
    if (lane == 0) pl->ver_n[(size_t)u * dm->vmax + v] = (float)cnt;
    return v;
  }
};

__global__ void __launch_bounds__(32) k_engine(Dims dm, Plan pl, CallArgs ca) {
  Eng e;
  e.dm = &dm;
  e.pl = &pl;
  e.ca = &ca;
  e.u = blockIdx.x;
  e.lane = threadIdx.x;
  e.C = dm.C;
  e.D = dm.D;
  const int u = e.u, lane = e.lane, C = dm.C, D = dm.D, M = dm.M;
  const dla_cache &cc = ca.cache;
  e.order = cc.order + (size_t)u * C;
  e.n = cc.n + (size_t)u * C;
  e.ts = cc.ts + (size_t)u * C;
  e.z = cc.z + (size_t)u * C * D;
  e.loss = cc.pair_loss + (size_t)u * C;
  e.slot_ver = pl.slot_ver + (size_t)u * C;
  e.ops = pl.ops + (size_t)u * dm.opsmax;
  e.nops = 0;
  e.nver = 0;
  e.m = cc.m[u];
  const int64_t t0 = cc.t[u];
  for (int w = 0; w < 4; w++) e.used[w] = 0;
  for (int p = 0; p < e.m; p++) {
    const int s = e.order[p];
    e.used[s >> 5] |= 1u << (s & 31);
  }
  for (int s = lane; s < C; s += 32) e.slot_ver[s] = -1;
  __syncwarp();

  const int nseg = pl.nseg[u];
  const int32_t *ss = pl.seg_start + (size_t)u * (dm.W + 1);
  const uint8_t *bflag = pl.b + (size_t)u * dm.W;
  const double *zend = pl.z_end + (size_t)u * dm.W * D;
  int32_t *tm0 = pl.tile_m0 + (size_t)u * dm.tiles;
  int32_t *tat = pl.tile_atoms + (size_t)u * dm.tiles * dm.amax;
  int32_t *tnev = pl.tile_nev + (size_t)u * dm.tiles;
  int32_t *toff = pl.tile_ev_off + (size_t)u * dm.tiles * M;
  int32_t *tmrg = pl.tile_ev_mrg + (size_t)u * dm.tiles * M;
  const bool tracing = ca.trace.merge_count != nullptr;
  int mcount = tracing ? ca.trace.merge_count[u] : 0;

  int j = 0;
  int cur_from = 0;  // first window token not yet added to the open state
  for (int c = 0; c < dm.tiles && c * M < ca.Tw; c++) {
    const int T0 = c * M;
    const int Tend = min(T0 + M, ca.Tw);
    // ---- states present just before the tile ----------------------------
    if (e.m > 0) {
      const int os = e.order[e.m - 1];
      if (T0 > cur_from) {
        e.emit(OP_ADD, os, cur_from, T0 - cur_from);
        if (lane == 0) e.n[os] += T0 - cur_from;
        __syncwarp();
        cur_from = T0;
      }
    }
    const int m0 = e.m;
    for (int p = 0; p < m0; p++) {
      const int slot = e.order[p];
      int v;
      if (p == m0 - 1) {  // open state: snapshot of its partial sum
        const double *zs = c == 0 ? e.z + (size_t)slot * D
                                  : pl.z_tile + ((size_t)u * dm.tiles + c) * D;
        v = e.new_version(slot, zs, e.n[slot]);
      } else {
        v = e.slot_ver[slot];
        if (v < 0) {
          v = e.new_version(slot, e.z + (size_t)slot * D, e.n[slot]);
          if (lane == 0) e.slot_ver[slot] = v;
        }
      }
      if (lane == 0) tat[(size_t)c * dm.amax + p] = v;
      __syncwarp();
    }
    if (lane == 0) tm0[c] = m0;
    // ---- boundaries inside the tile --------------------------------------
    int nev = 0;
    while (j < nseg && ss[j] < Tend) {
      const int s = ss[j];
      if (!(s == 0 && bflag[0] == 0)) {
        int mrg = EV_NO_MERGE;
        if (e.m > 0) {
          const int os = e.order[e.m - 1];
          if (s > cur_from) {
            e.emit(OP_ADD, os, cur_from, s - cur_from);
            if (lane == 0) e.n[os] += s - cur_from;
          }
          if (j >= 1)
            for (int cc2 = lane; cc2 < D; cc2 += 32) e.z[(size_t)os * D + cc2] = zend[(size_t)(j - 1) * D + cc2];
          __syncwarp();
          // seal: the open state joins the sealed list (all m states sealed)
          if (e.m >= 2) {
            const double l = e.ward(e.order[e.m - 2], e.order[e.m - 1]);
            if (lane == 0) e.loss[e.m - 2] = l;
          }
          __syncwarp();
          if (e.m == C) {
            // leftmost argmin over the C-1 sealed pairs
            double best = INFINITY;
            int bi = 0x7fffffff;
            for (int p = lane; p < C - 1; p += 32) {
              const double l = e.loss[p];
              if (l < best) {
                best = l;
                bi = p;
              }
            }
            for (int off = 16; off; off >>= 1) {
              const double ob = __shfl_down_sync(FULL, best, off);
              const int oi = __shfl_down_sync(FULL, bi, off);
              if (ob < best || (ob == best && oi < bi)) {
                best = ob;
                bi = oi;
              }
            }
            const int is = __shfl_sync(FULL, bi, 0);
            const int a = e.order[is], bb = e.order[is + 1];
            for (int cc2 = lane; cc2 < D; cc2 += 32)
              e.z[(size_t)a * D + cc2] = __dadd_rn(e.z[(size_t)a * D + cc2], e.z[(size_t)bb * D + cc2]);
            if (lane == 0) {
              e.n[a] += e.n[bb];
              e.slot_ver[a] = -1;
              e.slot_ver[bb] = -1;
            }
            e.emit(OP_MERGE, a, bb, 0);
            e.free_slot(bb);
            // drop position is+1 from order and pair (is) from the losses
            int32_t ov[4];
            double lv[4];
            for (int q = 0; q < 4; q++) {
              const int p = lane + 32 * q;
              ov[q] = (p >= is + 1 && p + 1 < C) ? e.order[p + 1] : 0;
              lv[q] = (p >= is + 1 && p + 1 < C - 1) ? e.loss[p + 1] : 0.0;
            }
            __syncwarp();
            for (int q = 0; q < 4; q++) {
              const int p = lane + 32 * q;
              if (p >= is + 1 && p + 1 < C) e.order[p] = ov[q];
              if (p >= is + 1 && p + 1 < C - 1) e.loss[p] = lv[q];
            }
            __syncwarp();
            e.m -= 1;  // C - 1 sealed
            if (is >= 1) {
              const double l = e.ward(e.order[is - 1], e.order[is]);
              if (lane == 0) e.loss[is - 1] = l;
            }
            if (is + 1 <= e.m - 1) {
              const double l = e.ward(e.order[is], e.order[is + 1]);
              if (lane == 0) e.loss[is] = l;
            }
            __syncwarp();
            mrg = is;
            if (tracing) {
              if (mcount < ca.trace.cap) {
                if (lane == 0) {
                  ca.trace.merge_t[(size_t)u * ca.trace.cap + mcount] = (int32_t)(t0 + s);
                  ca.trace.merge_i[(size_t)u * ca.trace.cap + mcount] = is;
                }
              } else if (lane == 0) {
                set_status(ca.dev_status, DLA_ERR_TRACE_OVERFLOW);
              }
              mcount++;
            }
          }
        }
        // open a new state at s
        const int slot = e.alloc_slot();
        e.emit(OP_ZERO, slot, 0, 0);
        for (int cc2 = lane; cc2 < D; cc2 += 32) e.z[(size_t)slot * D + cc2] = 0.0;
        if (lane == 0) {
          e.n[slot] = 0;
          e.ts[slot] = t0 + s;
          e.order[e.m] = slot;
          e.slot_ver[slot] = -1;
          toff[(size_t)c * M + nev] = s - T0;
          tmrg[(size_t)c * M + nev] = mrg;
        }
        __syncwarp();
        e.m += 1;
        cur_from = s;
        nev++;
      }
      j++;
    }
    if (lane == 0) tnev[c] = nev;
  }
  // ---- window end -------------------------------------------------------
  if (e.m > 0) {
    const int os = e.order[e.m - 1];
    if (ca.Tw > cur_from) {
      e.emit(OP_ADD, os, cur_from, ca.Tw - cur_from);
      if (lane == 0) e.n[os] += ca.Tw - cur_from;
    }
    for (int cc2 = lane; cc2 < D; cc2 += 32) e.z[(size_t)os * D + cc2] = zend[(size_t)(nseg - 1) * D + cc2];
  }
  if (lane == 0) {
    cc.m[u] = e.m;
    cc.t[u] = t0 + ca.Tw;
    cc.prev_r[u] = pl.r[(size_t)u * dm.W + ca.Tw - 1];
    pl.nops[u] = min(e.nops, dm.opsmax);
    if (tracing) ca.trace.merge_count[u] = mcount;
  }
  const size_t krow = ((size_t)u * dm.T + ca.w0 + ca.Tw - 1) * D;
  for (int cc2 = lane; cc2 < D; cc2 += 32) cc.prev_k[(size_t)u * D + cc2] = load_in(ca.k, ca.in_dtype, krow + cc2);
}

}  // namespace

cudaError_t launch_score(const Dims &dm, const Plan &pl, const CallArgs &ca, int policy,
                         cudaStream_t s) {
  dim3 g((ca.Tw + 255) / 256, dm.heads);
  k_score<<<g, 256, 0, s>>>(dm, pl, ca, policy);
  return cudaGetLastError();
}

cudaError_t launch_segscan(const Dims &dm, const Plan &pl, const CallArgs &ca, cudaStream_t s) {
  k_segscan<<<dm.heads, 1024, 0, s>>>(dm, pl, ca);
  return cudaGetLastError();
}

cudaError_t launch_segsum(const Dims &dm, const Plan &pl, const CallArgs &ca, cudaStream_t s) {
  dim3 g(64, dm.heads);
  k_segsum<<<g, dm.D, 0, s>>>(dm, pl, ca);
  return cudaGetLastError();
}

cudaError_t launch_engine(const Dims &dm, const Plan &pl, const CallArgs &ca, cudaStream_t s) {
  k_engine<<<dm.heads, 32, 0, s>>>(dm, pl, ca);
  return cudaGetLastError();
}

}  // namespace dla
