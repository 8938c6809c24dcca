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

constexpr int SCORE_TOK = 128;  // tokens per block

// Element c of a staged key row: rows hold the raw input (bf16 bits or fp32)
// with a row stride of `ld` 32-bit words (one pad word keeps thread t, which
// reads row t, on its own bank).
template <bool BF16>
__device__ __forceinline__ double key_at(const uint32_t *row, int c) {
  if (BF16) {
    const uint32_t w = row[c >> 1];
    return (double)__uint_as_float((c & 1) ? (w & 0xFFFF0000u) : (w << 16));
  }
  return (double)__uint_as_float(row[c]);
}

// Each token's squared norm is summed once and reused by the next token; dot
// and norm run as two independent chains, each in index order with explicit
// round-to-nearest (the oracle's operation sequence):
// cos = dot / (sqrt(|a|^2) * sqrt(|b|^2)), a zero norm gives r = 1.
template <bool BF16>
__device__ __forceinline__ void dot_norm(const uint32_t *a, const uint32_t *b, int D, double &dot,
                                         double &na) {
  dot = 0.0;
  na = 0.0;
  for (int c = 0; c < D; c++) {
    const double x = key_at<BF16>(a, c), y = key_at<BF16>(b, c);
    dot = __dadd_rn(dot, __dmul_rn(x, y));
    na = __dadd_rn(na, __dmul_rn(x, x));
  }
}
template <bool BF16>
__device__ __forceinline__ double norm2(const uint32_t *a, int D) {
  double n = 0.0;
  for (int c = 0; c < D; c++) {
    const double x = key_at<BF16>(a, c);
    n = __dadd_rn(n, __dmul_rn(x, x));
  }
  return n;
}
__device__ __forceinline__ double score_of(double dot, double na, double nb) {
  if (na == 0.0 || nb == 0.0) return 1.0;
  return __dsub_rn(1.0, __ddiv_rn(dot, __dmul_rn(__dsqrt_rn(na), __dsqrt_rn(nb))));
}

// Block of SCORE_TOK tokens; key rows of window tokens tb-2 .. tb+127 are
// staged with 16-byte loads (row tb-1 < 0 is the cache's previous key).
template <bool BF16>
__global__ void __launch_bounds__(SCORE_TOK) k_score(Dims dm, Plan pl, CallArgs ca, int policy) {
  extern __shared__ uint32_t srow[];  // [(SCORE_TOK + 2)][ld]
  const int u = blockIdx.y;
  const int tb = blockIdx.x * SCORE_TOK;
  const int tl = tb + threadIdx.x;
  const int D = dm.D;
  const int wpr = BF16 ? D / 2 : D;  // 32-bit words per row
  const int ld = wpr + 1;
  const int64_t t0 = ca.cache.t[u];
  __shared__ double rs[SCORE_TOK + 1];
  __shared__ double nsq[SCORE_TOK + 1];  // squared norm of token tb-1+i
  double r = 0.0;
  if (policy == DLA_POLICY_DYNAMIC) {
    const int vpr = wpr / 4;  // 16-byte vectors per row
    const uint4 *kv = reinterpret_cast<const uint4 *>(
        static_cast<const char *>(ca.k) + ((size_t)u * dm.T + ca.w0) * D * (BF16 ? 2 : 4));
#pragma unroll 4
    for (int e = threadIdx.x; e < (SCORE_TOK + 2) * vpr; e += SCORE_TOK) {
      const int rr = e / vpr, cv = e % vpr;
      const int t = tb - 2 + rr;
      if (t == -1) continue;  // the cache's previous key, written below
      uint4 x = make_uint4(0, 0, 0, 0);
      if (t >= 0 && t < ca.Tw) x = kv[(size_t)t * vpr + cv];
      uint32_t *dst = srow + rr * ld + cv * 4;
      dst[0] = x.x;
      dst[1] = x.y;
      dst[2] = x.z;
      dst[3] = x.w;
    }
    if (tb == 0) {  // row 1 = token -1 = the cache's previous key (fp32 values)
      for (int c = threadIdx.x; c < D; c += SCORE_TOK) {
        const float f = ca.cache.prev_k[(size_t)u * D + c];
        if (BF16) {
          const uint32_t hb = __float_as_uint(f) >> 16;  // exact: prev_k holds a bf16 value
          uint16_t *h = reinterpret_cast<uint16_t *>(srow + 1 * ld);
          h[c] = (uint16_t)hb;
        } else {
          srow[1 * ld + c] = __float_as_uint(f);
        }
      }
    }
    __syncthreads();
    double dot = 0.0, na = 0.0;
    if (tl < ca.Tw) dot_norm<BF16>(srow + (threadIdx.x + 2) * ld, srow + (threadIdx.x + 1) * ld, D, dot, na);
    nsq[threadIdx.x + 1] = na;
    if (threadIdx.x == 32) {  // a thread of the second warp: token tb-1
      const int tp = tb - 1;
      if (tp < 0) {
        nsq[0] = norm2<BF16>(srow + 1 * ld, D);
        rs[0] = ca.cache.prev_r[u];
      } else {
        double dp, np;
        dot_norm<BF16>(srow + 1 * ld, srow + 0 * ld, D, dp, np);
        nsq[0] = np;
        rs[0] = (t0 + tp == 0) ? 0.0 : score_of(dp, np, norm2<BF16>(srow + 0 * ld, D));
      }
    }
    __syncthreads();
    if (tl < ca.Tw) r = (t0 + tl == 0) ? 0.0 : score_of(dot, na, nsq[threadIdx.x]);
  }
  rs[threadIdx.x + 1] = r;
  __syncthreads();
  if (tl >= ca.Tw) return;
  uint8_t b = 1;
  if (policy == DLA_POLICY_DYNAMIC) {
    const double rp = rs[threadIdx.x];
    const double tau = (double)ca.tau;
    const bool join = (t0 + tl > 0) && (r < tau) && (rp < tau);
    b = join ? 0 : 1;
  }
  pl.r[(size_t)u * dm.W + tl] = r;
  pl.b[(size_t)u * dm.W + tl] = b;
  if (ca.trace.boundary) ca.trace.boundary[(size_t)u * dm.T + ca.w0 + tl] = b;
}

// phi(x) in fp64 for every bf16 bit pattern (same exp as inline evaluation).
__global__ void k_phi_table(double *tab) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < 65536) tab[i] = phi64((double)__uint_as_float((uint32_t)i << 16));
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

// z = sum of phi(k) of every window piece, in fp64, in two levels:
//   k_tilesum    per (head, tile): token-order sums of each run of the tile's
//                tokens between boundaries ("part"), stored at the part's first
//                token;
//   k_segcombine per segment: its parts added in time order (the cache's z
//                of a continued open state first), writing the segment's end
//                sum and the open state's partial sum before each tile.
// Each dependent fp64 chain is at most a tile (128 tokens) or the tiles a
// segment spans; the association differs from a strict token-order sum by
// rounding only (merge choices are then the same unless two Ward losses tie
// to within rounding).
__global__ void k_tilesum(Dims dm, Plan pl, CallArgs ca) {
  const int u = blockIdx.y, tile = blockIdx.x;
  const int c = threadIdx.x;  // dimension
  const int D = dm.D, M = dm.M;
  const int T0 = tile * M;
  if (T0 >= ca.Tw) return;
  const int T1 = min(T0 + M, ca.Tw);
  const uint8_t *b = pl.b + (size_t)u * dm.W;
  const size_t kb = ((size_t)u * dm.T + ca.w0) * D + c;
  double *zp = pl.z_part + (size_t)u * dm.W * D + c;
  const double *__restrict__ tab = pl.phi_tab;
  constexpr int CH = 16;
  double z = 0.0;
  int part = T0;
  for (int s0 = T0; s0 < T1; s0 += CH) {
    double ph[CH];
#pragma unroll
    for (int i = 0; i < CH; i++) {
      const int s = s0 + i;
      const float x = s < T1 ? load_in(ca.k, ca.in_dtype, kb + (size_t)s * D) : 0.f;
      ph[i] = tab ? __ldg(tab + (__float_as_uint(x) >> 16)) : phi64((double)x);
    }
#pragma unroll
    for (int i = 0; i < CH; i++) {
      const int s = s0 + i;
      if (s < T1) {
        if (s > T0 && b[s]) {
          zp[(size_t)part * D] = z;
          part = s;
          z = 0.0;
        }
        z = __dadd_rn(z, ph[i]);
      }
    }
  }
  zp[(size_t)part * D] = z;
}

__global__ void k_segcombine(Dims dm, Plan pl, CallArgs ca) {
  const int u = blockIdx.y;
  const int c = threadIdx.x;  // dimension
  const int D = dm.D, M = dm.M;
  const int nseg = pl.nseg[u];
  const int32_t *ss = pl.seg_start + (size_t)u * (dm.W + 1);
  const uint8_t *b = pl.b + (size_t)u * dm.W;
  const double *zp = pl.z_part + (size_t)u * dm.W * D + c;
  for (int j = blockIdx.x; j < nseg; j += gridDim.x) {
    const int s0 = ss[j];
    const int s1 = j + 1 < nseg ? ss[j + 1] : ca.Tw;
    double z = 0.0;
    if (j == 0 && b[0] == 0) {
      // continuation of the cache's open state
      const int m = ca.cache.m[u];
      const int os = ca.cache.order[(size_t)u * dm.C + m - 1];
      z = ca.cache.z[((size_t)u * dm.C + os) * D + c];
    }
    z = __dadd_rn(z, zp[(size_t)s0 * D]);
    for (int T0 = (s0 / M + 1) * M; T0 < s1; T0 += M) {
      pl.z_tile[((size_t)u * dm.tiles + T0 / M) * D + c] = z;
      z = __dadd_rn(z, zp[(size_t)T0 * D]);
    }
    // the tile start right after the segment's end (if the segment ends at a
    // tile boundary the next tile's open state is this one, complete)
    if (s1 % M == 0 && s1 < ca.Tw) pl.z_tile[((size_t)u * dm.tiles + s1 / M) * D + c] = z;
    pl.z_end[((size_t)u * dm.W + j) * D + c] = z;
  }
}

// ---------------------------------------------------------------- engine ----
// One warp per head.  The head's cache summaries (order, n, ts, version of
// each slot, pair losses and the fp64 z of every slot) live in shared memory
// for the whole window and are written back at its end.

struct EngSmem {
  int32_t order[128];
  int32_t sver[128];
  long long n[128];
  long long ts[128];
  double loss[128];
  double z[1];  // [C][D], dynamic
};

struct Eng {
  const Dims *dm;
  const Plan *pl;
  const CallArgs *ca;
  EngSmem *sm;
  int u, lane, C, D;
  int4 *ops;
  int nops, nver, m, npieces;
  uint32_t used[4];

  __device__ double *zs(int slot) const { return sm->z + (size_t)slot * D; }
  // lane-local emit at position nops + rank; the caller advances nops
  __device__ void put(int idx, int op, int a, int b, int c) const {
    if (idx < dm->opsmax) ops[idx] = make_int4(op, a, b, c);
    else set_status(ca->dev_status, DLA_ERR_INVARIANT);
  }
  __device__ void emit(int op, int a, int b, int c) {
    if (lane == 0) put(nops, op, a, b, c);
    nops++;
  }
  // tokens [from, from + cnt) join the open state `slot`: a tensor-core piece
  // when long enough (and the path has pieces), else SIMT rank-1 adds
  __device__ void emit_add(int slot, int from, int cnt) {
    if (dm->pmax > 0 && cnt >= PIECE_MIN) {
      if (npieces >= dm->pmax && lane == 0) set_status(ca->dev_status, DLA_ERR_INVARIANT);
      emit(OP_ADDP, slot, npieces, cnt);
      npieces++;
    } else {
      emit(OP_ADD, slot, from, cnt);
    }
  }
  // Ward loss with one reciprocal per state: mu = z * (1 / n) (within an ulp
  // of z / n; merge choices agree with the oracle whenever the best and
  // second-best losses differ by more than rounding)
  __device__ double ward(int sa, int sb) const {
    const double na = (double)sm->n[sa], nb = (double)sm->n[sb];
    const double ia = __drcp_rn(na), ib = __drcp_rn(nb);
    const double *za = zs(sa), *zb = zs(sb);
    double s = 0.0;
    for (int c = lane; c < D; c += 32) {
      const double diff = __dsub_rn(__dmul_rn(za[c], ia), __dmul_rn(zb[c], ib));
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
        const int slot = w * 32 + __ffs(freeb) - 1;
        if (slot < C) {
          used[w] |= 1u << (slot & 31);
          return slot;
        }
      }
    }
    if (lane == 0) set_status(ca->dev_status, DLA_ERR_INVARIANT);
    return 0;
  }
  __device__ void free_slot(int s) { used[s >> 5] &= ~(1u << (s & 31)); }
  // the same from per-lane registers (dimension lane + 32 q)
  __device__ void write_mu_regs(int v, const double *zr, long long cnt) const {
    float *zv = pl->ver_z + ((size_t)u * dm->vmax + v) * D;
#pragma unroll
    for (int q = 0; q < 4; q++)
      if (lane + 32 * q < D) zv[lane + 32 * q] = (float)zr[q];
    if (lane == 0) pl->ver_n[(size_t)u * dm->vmax + v] = (float)cnt;
  }
  // phi(k) sum and count of version v (all lanes); readouts divide
  __device__ void write_mu(int v, const double *zsrc, long long cnt) const {
    float *zv = pl->ver_z + ((size_t)u * dm->vmax + v) * D;
    for (int c = lane; c < D; c += 32) zv[c] = (float)zsrc[c];
    if (lane == 0) pl->ver_n[(size_t)u * dm->vmax + v] = (float)cnt;
  }
};

__global__ void __launch_bounds__(32) k_engine(Dims dm, Plan pl, CallArgs ca) {
  extern __shared__ __align__(16) unsigned char eng_raw[];
  EngSmem *sm = reinterpret_cast<EngSmem *>(eng_raw);
  Eng e;
  e.dm = &dm;
  e.pl = &pl;
  e.ca = &ca;
  e.sm = sm;
  e.u = blockIdx.x;
  e.lane = threadIdx.x;
  e.C = dm.C;
  e.D = dm.D;
  const int u = e.u, lane = e.lane, C = dm.C, D = dm.D, M = dm.M;
  const dla_cache &cc = ca.cache;
  // ---- load the head's summaries ------------------------------------------
  for (int p = lane; p < C; p += 32) {
    sm->order[p] = cc.order[(size_t)u * C + p];
    sm->n[p] = cc.n[(size_t)u * C + p];
    sm->ts[p] = cc.ts[(size_t)u * C + p];
    sm->loss[p] = cc.pair_loss[(size_t)u * C + p];
    sm->sver[p] = -1;
  }
  for (int i = lane; i < C * D; i += 32) sm->z[i] = cc.z[(size_t)u * C * D + i];
  __syncwarp();
  e.ops = pl.ops + (size_t)u * dm.opsmax;
  e.nops = 0;
  e.nver = 0;
  e.npieces = 0;
  e.m = cc.m[u];
  const int64_t t0 = cc.t[u];
  for (int w = 0; w < 4; w++) e.used[w] = 0;
  for (int p = 0; p < e.m; p++) {
    const int s = sm->order[p];
    e.used[s >> 5] |= 1u << (s & 31);
  }
  if (e.m > 0) e.emit(OP_LOAD, sm->order[e.m - 1], 0, 0);

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
  // one step of look-ahead on global reads: the next boundary positions, the
  // end sum of the segment sealed at the next boundary, the next tile's
  // open-state partial sum
  int ss_cur = nseg > 0 ? ss[0] : 0x7fffffff;
  int ss_nxt = nseg > 1 ? ss[1] : 0x7fffffff;
  double zprev[4] = {0.0, 0.0, 0.0, 0.0};  // end sum of segment j-1
  double ztile[4] = {0.0, 0.0, 0.0, 0.0};  // open-state partial sum before tile c
  for (int c = 0; c < dm.tiles && c * M < ca.Tw; c++) {
    const int T0 = c * M;
    const int Tend = min(T0 + M, ca.Tw);
    double ztile_cur[4];
#pragma unroll
    for (int q = 0; q < 4; q++) ztile_cur[q] = ztile[q];
#pragma unroll
    for (int q = 0; q < 4; q++)
      ztile[q] = (c + 1 < dm.tiles && (c + 1) * M < ca.Tw && lane + 32 * q < D)
                     ? pl.z_tile[((size_t)u * dm.tiles + c + 1) * D + lane + 32 * q] : 0.0;
    // ---- states present just before the tile ----------------------------
    if (e.m > 0) {
      const int os = sm->order[e.m - 1];
      if (T0 > cur_from) {
        e.emit_add(os, cur_from, T0 - cur_from);
        if (lane == 0) sm->n[os] += T0 - cur_from;
        __syncwarp();
        cur_from = T0;
      }
    }
    if (lane == 0 && dm.pmax > 0) pl.tile_pbase[(size_t)u * dm.tiles + c] = e.npieces;
    const int m0 = e.m;
    for (int p0 = 0; p0 < m0; p0 += 32) {
      const int p = p0 + lane;
      const int slot = p < m0 ? sm->order[p] : 0;
      const bool need = p < m0 && (p == m0 - 1 || sm->sver[slot] < 0);
      const unsigned bal = __ballot_sync(FULL, need);
      const int rank = __popc(bal & ((1u << lane) - 1u));
      if (need) {
        const int v = e.nver + rank;
        e.put(e.nops + rank, OP_SHADOW, slot, v, 0);
        if (p != m0 - 1) sm->sver[slot] = v;
        tat[(size_t)c * dm.amax + p] = v;
      } else if (p < m0) {
        tat[(size_t)c * dm.amax + p] = sm->sver[slot];
      }
      // means of the new versions (lanes over dimensions)
      unsigned todo = bal;
      while (todo) {
        const int l = __ffs(todo) - 1;
        todo &= todo - 1;
        const int pv = p0 + l;
        const int sl = sm->order[pv];
        const int v = e.nver + __popc(bal & ((1u << l) - 1u));
        if (pv == m0 - 1 && c > 0) e.write_mu_regs(v, ztile_cur, sm->n[sl]);
        else e.write_mu(v, e.zs(sl), sm->n[sl]);
      }
      e.nver += __popc(bal);
      e.nops += __popc(bal);
      __syncwarp();
    }
    if (e.nver > dm.vmax && lane == 0) set_status(ca.dev_status, DLA_ERR_INVARIANT);
    if (lane == 0) tm0[c] = m0;
    // ---- boundaries inside the tile --------------------------------------
    int nev = 0;
    while (j < nseg && ss_cur < Tend) {
      const int s = ss_cur;
      const int ss_n2 = j + 2 < nseg ? ss[j + 2] : 0x7fffffff;
      double znext[4];
#pragma unroll
      for (int q = 0; q < 4; q++) znext[q] = lane + 32 * q < D ? zend[(size_t)j * D + lane + 32 * q] : 0.0;
      if (!(s == 0 && bflag[0] == 0)) {
        int mrg = EV_NO_MERGE;
        if (e.m > 0) {
          const int os = sm->order[e.m - 1];
          if (s > cur_from) {
            e.emit_add(os, cur_from, s - cur_from);
            if (lane == 0) sm->n[os] += s - cur_from;
          }
          e.emit(OP_STORE, os, 0, 0);
          if (j >= 1) {
#pragma unroll
            for (int q = 0; q < 4; q++)
              if (lane + 32 * q < D) e.zs(os)[lane + 32 * q] = zprev[q];
          }
          __syncwarp();
          // seal: the open state joins the sealed list (all m states sealed)
          if (e.m >= 2) {
            const double l = e.ward(sm->order[e.m - 2], sm->order[e.m - 1]);
            if (lane == 0) sm->loss[e.m - 2] = l;
          }
          __syncwarp();
          if (e.m == C) {
            // leftmost argmin over the C-1 sealed pairs
            double best = INFINITY;
            int bi = 0x7fffffff;
            for (int p = lane; p < C - 1; p += 32) {
              const double l = sm->loss[p];
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
            const int a = sm->order[is], bb = sm->order[is + 1];
            for (int d2 = lane; d2 < D; d2 += 32) e.zs(a)[d2] = __dadd_rn(e.zs(a)[d2], e.zs(bb)[d2]);
            if (lane == 0) {
              sm->n[a] += sm->n[bb];
              sm->sver[a] = -1;
              sm->sver[bb] = -1;
            }
            e.emit(OP_MERGE, a, bb, 0);
            e.free_slot(bb);
            // drop position is+1 from order and pair (is) from the losses
            int32_t ov[4];
            double lv[4];
            for (int q = 0; q < 4; q++) {
              const int p = lane + 32 * q;
              ov[q] = (p >= is + 1 && p + 1 < C) ? sm->order[p + 1] : 0;
              lv[q] = (p >= is + 1 && p + 1 < C - 1) ? sm->loss[p + 1] : 0.0;
            }
            __syncwarp();
            for (int q = 0; q < 4; q++) {
              const int p = lane + 32 * q;
              if (p >= is + 1 && p + 1 < C) sm->order[p] = ov[q];
              if (p >= is + 1 && p + 1 < C - 1) sm->loss[p] = lv[q];
            }
            __syncwarp();
            e.m -= 1;  // C - 1 sealed
            if (is >= 1) {
              const double l = e.ward(sm->order[is - 1], sm->order[is]);
              if (lane == 0) sm->loss[is - 1] = l;
            }
            if (is + 1 <= e.m - 1) {
              const double l = e.ward(sm->order[is], sm->order[is + 1]);
              if (lane == 0) sm->loss[is] = l;
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
        for (int d2 = lane; d2 < D; d2 += 32) e.zs(slot)[d2] = 0.0;
        if (lane == 0) {
          sm->n[slot] = 0;
          sm->ts[slot] = t0 + s;
          sm->order[e.m] = slot;
          sm->sver[slot] = -1;
          toff[(size_t)c * M + nev] = s - T0;
          tmrg[(size_t)c * M + nev] = mrg;
        }
        __syncwarp();
        e.m += 1;
        cur_from = s;
        nev++;
      }
#pragma unroll
      for (int q = 0; q < 4; q++) zprev[q] = znext[q];
      ss_cur = ss_nxt;
      ss_nxt = ss_n2;
      j++;
    }
    if (lane == 0) tnev[c] = nev;
  }
  // ---- window end -------------------------------------------------------
  if (e.m > 0) {
    const int os = sm->order[e.m - 1];
    if (ca.Tw > cur_from) {
      e.emit_add(os, cur_from, ca.Tw - cur_from);
      if (lane == 0) sm->n[os] += ca.Tw - cur_from;
    }
    e.emit(OP_STORE, os, 0, 0);
    for (int d2 = lane; d2 < D; d2 += 32) e.zs(os)[d2] = zend[(size_t)(nseg - 1) * D + d2];
  }
  __syncwarp();
  for (int p = lane; p < C; p += 32) {
    cc.order[(size_t)u * C + p] = sm->order[p];
    cc.n[(size_t)u * C + p] = sm->n[p];
    cc.ts[(size_t)u * C + p] = sm->ts[p];
    cc.pair_loss[(size_t)u * C + p] = sm->loss[p];
  }
  for (int i = lane; i < C * D; i += 32) cc.z[(size_t)u * C * D + i] = sm->z[i];
  if (lane == 0) {
    cc.m[u] = e.m;
    cc.t[u] = t0 + ca.Tw;
    cc.prev_r[u] = pl.r[(size_t)u * dm.W + ca.Tw - 1];
    pl.nops[u] = min(e.nops, dm.opsmax);
    if (tracing) ca.trace.merge_count[u] = mcount;
  }
  const size_t krow = ((size_t)u * dm.T + ca.w0 + ca.Tw - 1) * D;
  for (int d2 = lane; d2 < D; d2 += 32) cc.prev_k[(size_t)u * D + d2] = load_in(ca.k, ca.in_dtype, krow + d2);
}

}  // namespace

cudaError_t launch_score(const Dims &dm, const Plan &pl, const CallArgs &ca, int policy,
                         cudaStream_t s) {
  const bool bf = ca.in_dtype == DLA_BF16;
  const size_t sb = sizeof(uint32_t) * (SCORE_TOK + 2) * ((bf ? dm.D / 2 : dm.D) + 1);
  dim3 g((ca.Tw + SCORE_TOK - 1) / SCORE_TOK, dm.heads);
  if (bf) {
    cudaError_t e = cudaFuncSetAttribute(k_score<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sb);
    if (e != cudaSuccess) return e;
    k_score<true><<<g, SCORE_TOK, sb, s>>>(dm, pl, ca, policy);
  } else {
    cudaError_t e = cudaFuncSetAttribute(k_score<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sb);
    if (e != cudaSuccess) return e;
    k_score<false><<<g, SCORE_TOK, sb, s>>>(dm, pl, ca, policy);
  }
  return cudaGetLastError();
}

cudaError_t launch_phi_table(double *tab, cudaStream_t s) {
  k_phi_table<<<256, 256, 0, s>>>(tab);
  return cudaGetLastError();
}

cudaError_t launch_segscan(const Dims &dm, const Plan &pl, const CallArgs &ca, cudaStream_t s) {
  k_segscan<<<dm.heads, 1024, 0, s>>>(dm, pl, ca);
  return cudaGetLastError();
}

cudaError_t launch_segsum(const Dims &dm, const Plan &pl, const CallArgs &ca, cudaStream_t s) {
  k_tilesum<<<dim3(dm.tiles, dm.heads), dm.D, 0, s>>>(dm, pl, ca);
  k_segcombine<<<dim3(64, dm.heads), dm.D, 0, s>>>(dm, pl, ca);
  return cudaGetLastError();
}

cudaError_t launch_engine(const Dims &dm, const Plan &pl, const CallArgs &ca, cudaStream_t s) {
  const size_t sb = sizeof(EngSmem) + sizeof(double) * ((size_t)dm.C * dm.D - 1);
  cudaError_t e = cudaFuncSetAttribute(k_engine, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sb);
  if (e != cudaSuccess) return e;
  k_engine<<<dm.heads, 32, sb, s>>>(dm, pl, ca);
  return cudaGetLastError();
}

}  // namespace dla
