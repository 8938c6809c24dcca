// decide.cu -- decision kernels of a DLA prefill window.
//
//   k_score    r_t = 1 - cos(k_t, k_{t-1}) in fp64 and the boundary flag
//              b_t = not (r_t < tau and r_{t-1} < tau), one thread per token
//              (ai-feeds.com "Dynamic Linear Attention" summary, section
//              信息感知的动态状态合并: a token joins only when it and its
//              predecessor are low-information; Chlience section 5.1: b_t = 1
//              opens a new state).
//   k_segscan  window pieces: {0} and every boundary t > 0 (warp ballots).
//   k_score    also writes the tile sums below for bf16 keys (its block of
//              128 tokens is then one readout tile);
//   k_tilesum_any  otherwise, per (tile, head): fp64 sum of phi(k) over each
//              run of a piece inside the tile, in token order.
//   k_segcombine  per piece: the runs' sums in time order (after the cached
//              open state's z for a continuation) give z at the piece's end
//              and the open state's partial z before each readout tile.
//   k_engine   one warp per head walks tiles and boundaries in time order:
//              seals, capacity merges by least Ward loss (Chlience section 5.2
//              and Corollary 1), slot allocation; emits the materializer op
//              list, the per-tile atoms/events and the merge trace.  Under the
//              information policy the pair criterion is the information
//              density (I_a + I_b) / (n_a + n_b) of the pair's score sums
//              (Chlience section 5.2) and the boundaries come from info.cu.
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
// The product of two bf16 (or fp32) values is exact in fp64, so
// fma(x, y, acc) rounds exactly like acc + x * y with the product rounded
// first: one fp64 operation per term instead of two.
template <bool BF16>
__device__ __forceinline__ void dot_norm(const uint32_t *a, const uint32_t *b, int D, double &dot,
                                         double &na) {
  dot = 0.0;
  na = 0.0;
  for (int c = 0; c < D; c++) {
    const double x = key_at<BF16>(a, c), y = key_at<BF16>(b, c);
    dot = __fma_rn(x, y, dot);
    na = __fma_rn(x, x, na);
  }
}
template <bool BF16>
__device__ __forceinline__ double norm2(const uint32_t *a, int D) {
  double n = 0.0;
  for (int c = 0; c < D; c++) {
    const double x = key_at<BF16>(a, c);
    n = __fma_rn(x, x, n);
  }
  return n;
}
__device__ __forceinline__ double score_of(double dot, double na, double nb) {
  if (na == 0.0 || nb == 0.0) return 1.0;
  return __dsub_rn(1.0, __ddiv_rn(dot, __dmul_rn(__dsqrt_rn(na), __dsqrt_rn(nb))));
}

// phi of a bf16 input in fp64.  Negative inputs need exp: those with a
// biased exponent in [PHI_E0, PHI_E0 + PHI_NE) (|x| in [2^-24, 16)) come from
// a table filled with the same exp() per call; other negatives call exp().
constexpr int PHI_E0 = 103, PHI_NE = 28, PHI_TAB = PHI_NE * 128;

__global__ void k_phi_table(double *tab) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < PHI_TAB) {
    const uint32_t bits = 0x8000u | ((uint32_t)(PHI_E0 + i / 128) << 7) | (uint32_t)(i % 128);
    tab[i] = phi64((double)__uint_as_float(bits << 16));
  }
}

__device__ __forceinline__ double phi_bf16_f64(uint32_t bits, const double *s_tab) {
  const float x = __uint_as_float(bits << 16);
  if (!(bits & 0x8000u)) return (double)x + 1.0;  // x >= +0 (phi(+0) = 1 either way)
  const uint32_t e = ((bits >> 7) & 0xFFu) - PHI_E0;
  return e < (uint32_t)PHI_NE ? s_tab[e * 128 + (bits & 127u)] : phi64((double)x);
}

// Block of SCORE_TOK tokens; key rows of window tokens tb-2 .. tb+127 are
// staged with 16-byte loads.  In a call's first window, row tb-1 < 0 is the
// cache's previous key and r of token -1 the cache's; later windows take both
// from the call's own input (the same fp64 sequence as the window before), so
// they need nothing the previous window's engine writes.
// With `sums` (bf16 keys, readout tiles of SCORE_TOK rows) the block, which is
// then one tile, also writes the tile's per-run sums of phi(k) from the
// staged rows.
template <bool BF16>
__global__ void __launch_bounds__(SCORE_TOK, 6) k_score(Dims dm, Plan pl, CallArgs ca, int policy,
                                                     int sums) {
  extern __shared__ uint32_t srow[];  // [(SCORE_TOK + 2)][ld]
  const int u = blockIdx.y;
  const int tb = blockIdx.x * SCORE_TOK;
  const int tl = tb + threadIdx.x;
  const int D = dm.D;
  const int Tw = tw_of(ca, u);  // this stream's tokens in the window
  if (tb >= Tw) return;         // (a whole block: a ragged stream ends before it)
  const int wpr = BF16 ? D / 2 : D;  // 32-bit words per row
  const int ld = wpr + 1;
  // the stream's token count before the window (read only in a call's first
  // window: later ones never hold the stream's first token)
  const int64_t t0 = ca.w0 == 0 ? ca.cache.t[u] : 1;
  __shared__ double rs[SCORE_TOK + 1];
  __shared__ double nsq[SCORE_TOK + 1];  // squared norm of token tb-1+i
  __shared__ uint8_t s_b[SCORE_TOK];
  double r = 0.0;
  if (policy == DLA_POLICY_DYNAMIC) {
    const int vpr = wpr / 4;  // 16-byte vectors per row
    const uint4 *kv = reinterpret_cast<const uint4 *>(
        static_cast<const char *>(ca.k) + ((size_t)u * dm.T + ca.w0) * D * (BF16 ? 2 : 4));
    if (BF16) {
      // the block's rows in two batches of 16-byte loads, each batch in flight
      // at once (at most 17 loads per thread for d = 128), then its stores
      // into the padded rows
      constexpr int MAXIT = ((SCORE_TOK + 2) * 16 + SCORE_TOK - 1) / SCORE_TOK;
      constexpr int BATCH = (MAXIT + 1) / 2;
#pragma unroll
      for (int b0 = 0; b0 < MAXIT; b0 += BATCH) {
        uint4 xs[BATCH];
#pragma unroll
        for (int i = 0; i < BATCH; i++) {
          const int e = threadIdx.x + (b0 + i) * SCORE_TOK;
          const int rr = e / vpr, cv = e % vpr;
          const int t = tb - 2 + rr;
          xs[i] = make_uint4(0, 0, 0, 0);
          if (b0 + i < MAXIT && e < (SCORE_TOK + 2) * vpr && ca.w0 + t >= 0 && t < Tw)
            xs[i] = kv[(ptrdiff_t)t * vpr + cv];
        }
#pragma unroll
        for (int i = 0; i < BATCH; i++) {
          const int e = threadIdx.x + (b0 + i) * SCORE_TOK;
          const int rr = e / vpr, cv = e % vpr;
          if (b0 + i >= MAXIT || e >= (SCORE_TOK + 2) * vpr || (tb - 2 + rr == -1 && ca.w0 == 0)) continue;
          uint32_t *dst = srow + rr * ld + cv * 4;
          dst[0] = xs[i].x;
          dst[1] = xs[i].y;
          dst[2] = xs[i].z;
          dst[3] = xs[i].w;
        }
      }
    } else {
#pragma unroll 4
      for (int e = threadIdx.x; e < (SCORE_TOK + 2) * vpr; e += SCORE_TOK) {
        const int rr = e / vpr, cv = e % vpr;
        const int t = tb - 2 + rr;
        if (t == -1 && ca.w0 == 0) continue;  // the cache's previous key, written below
        uint4 x = make_uint4(0, 0, 0, 0);
        if (ca.w0 + t >= 0 && t < Tw) x = kv[(ptrdiff_t)t * vpr + cv];
        uint32_t *dst = srow + rr * ld + cv * 4;
        dst[0] = x.x;
        dst[1] = x.y;
        dst[2] = x.z;
        dst[3] = x.w;
      }
    }
    if (tb == 0 && ca.w0 == 0) {  // row 1 = token -1 = the cache's previous key (fp32 values)
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
    if (tl < Tw) dot_norm<BF16>(srow + (threadIdx.x + 2) * ld, srow + (threadIdx.x + 1) * ld, D, dot, na);
    nsq[threadIdx.x + 1] = na;
    if (threadIdx.x == 32) {  // a thread of the second warp: token tb-1
      const int tp = tb - 1;
      if (tp < 0 && ca.w0 == 0) {
        nsq[0] = norm2<BF16>(srow + 1 * ld, D);
        rs[0] = ca.cache.prev_r[u];
      } else {
        double dp, np;
        dot_norm<BF16>(srow + 1 * ld, srow + 0 * ld, D, dp, np);
        nsq[0] = np;
        rs[0] = (ca.w0 == 0 && t0 + tp == 0) ? 0.0 : score_of(dp, np, norm2<BF16>(srow + 0 * ld, D));
      }
    }
    __syncthreads();
    if (tl < Tw) r = (ca.w0 == 0 && t0 + tl == 0) ? 0.0 : score_of(dot, na, nsq[threadIdx.x]);
  }
  rs[threadIdx.x + 1] = r;
  __syncthreads();
  uint8_t b = 1;
  if (tl < Tw) {
    if (policy == DLA_POLICY_DYNAMIC) {
      const double rp = rs[threadIdx.x];
      const double tau = (double)ca.tau;
      const bool join = (ca.w0 > 0 || t0 + tl > 0) && (r < tau) && (rp < tau);
      b = join ? 0 : 1;
    }
    pl.r[(size_t)u * dm.W + tl] = r;
    pl.b[(size_t)u * dm.W + tl] = b;
    if (ca.trace.boundary) ca.trace.boundary[(size_t)u * dm.T + ca.w0 + tl] = b;
  }
  if (!BF16 || !sums) return;
  // thread c: token-order fp64 sum of phi(k[.][c]) over each run of the tile
  // between boundaries, stored at the run's first token
  s_b[threadIdx.x] = b;
  __syncthreads();
  const int len = min(SCORE_TOK, Tw - tb);
  for (int c = threadIdx.x; c < D; c += SCORE_TOK) {
    double *zp = pl.z_part + (size_t)u * dm.W * D + c;
    double z = 0.0;
    int part = tb;
#pragma unroll 4
    for (int i = 0; i < len; i++) {
      if (i > 0 && s_b[i]) {
        zp[(size_t)part * D] = z;
        part = tb + i;
        z = 0.0;
      }
      const uint32_t w = srow[(i + 2) * ld + (c >> 1)];
      z = __dadd_rn(z, phi_bf16_f64((c & 1) ? (w >> 16) : (w & 0xFFFFu), pl.phi_tab));
    }
    zp[(size_t)part * D] = z;
  }
}

// phi(x) in fp64 for every bf16 bit pattern (same exp as inline evaluation).

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
  const int Tw = tw_of(ca, u);
  for (int c0 = 0; c0 < Tw; c0 += blockDim.x) {
    const int t = c0 + threadIdx.x;
    const bool f = t > 0 && t < Tw && b[t];
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
  if (threadIdx.x == 0) pl.nseg[u] = Tw > 0 ? base : 0;  // no token, no piece
}

// z = sum of phi(k) of every window piece, in fp64, in two levels:
//   tile sums    per (head, tile): token-order sums of each run of the tile's
//                tokens between boundaries ("part"), stored at the part's first
//                token (k_score for bf16 keys, else k_tilesum_any);
//   k_segcombine per segment: its parts added in time order (the cache's z
//                of a continued open state first), writing the segment's end
//                sum and the open state's partial sum before each tile.
// Each dependent fp64 chain is at most a tile (128 tokens) or the tiles a
// segment spans; the association differs from a strict token-order sum by
// rounding only (merge choices are then the same unless two Ward losses tie
// to within rounding).
// Tile sums of other inputs (fp32 keys, or tiles other than the score's
// blocks): direct loads, phi64.
__global__ void k_tilesum_any(Dims dm, Plan pl, CallArgs ca) {
  const int u = blockIdx.y, tile = blockIdx.x;
  const int c = threadIdx.x;  // dimension
  const int D = dm.D, M = dm.M;
  const int T0 = tile * M;
  const int Tw = tw_of(ca, u);
  if (T0 >= Tw) return;
  const int T1 = min(T0 + M, Tw);
  const uint8_t *b = pl.b + (size_t)u * dm.W;
  const size_t kb = ((size_t)u * dm.T + ca.w0) * D + c;
  double *zp = pl.z_part + (size_t)u * dm.W * D + c;
  double z = 0.0;
  int part = T0;
  for (int s = T0; s < T1; s++) {
    if (s > T0 && b[s]) {
      zp[(size_t)part * D] = z;
      part = s;
      z = 0.0;
    }
    z = __dadd_rn(z, phi64((double)load_in(ca.k, ca.in_dtype, kb + (size_t)s * D)));
  }
  zp[(size_t)part * D] = z;
}

__global__ void k_segcombine(Dims dm, Plan pl, CallArgs ca) {
  const int u = blockIdx.y;
  const int c = threadIdx.x;  // dimension
  const int D = dm.D, M = dm.M;
  const int nseg = pl.nseg[u];
  const int Tw = tw_of(ca, u);
  const int32_t *ss = pl.seg_start + (size_t)u * (dm.W + 1);
  const uint8_t *b = pl.b + (size_t)u * dm.W;
  const double *zp = pl.z_part + (size_t)u * dm.W * D + c;
  for (int j = blockIdx.x; j < nseg; j += gridDim.x) {
    const int s0 = ss[j];
    const int s1 = j + 1 < nseg ? ss[j + 1] : Tw;
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
    if (s1 % M == 0 && s1 < Tw) pl.z_tile[((size_t)u * dm.tiles + s1 / M) * D + c] = z;
    pl.z_end[((size_t)u * dm.W + j) * D + c] = z;
  }
}

// ---------------------------------------------------------------- engine ----
// One warp per head walks the window's tiles and segment starts in time order.
// Shared memory holds the head's cache summaries for the whole window (time
// order, counts, first times, versions, sealed-pair losses, 1/n of sealed
// states and the fp64 z of every slot) and a ring of segment-end sums z_end
// that asynchronous copies fill ZR segments ahead.  Lane l owns dimensions
// l, l + 32, ... of every z, so z updates need no warp synchronisation.
// Kernel parameters are copied to registers (no pointer to them is formed)
// and segment starts are prefetched 32 at a time into lane registers.

constexpr int ZR = 8;  // z_end ring depth

struct EngSmem {
  int32_t order[128];
  int32_t sver[128];
  int32_t lastmod[128];    // op that produced the slot's sealed value (-1: none)
  uint32_t used[4];
  long long n[128];
  long long ts[128];
  double loss[128];
  double rn[128];          // 1 / n of sealed states (__drcp_rn)
  double info[128];        // score sum of each slot's state (information policy)
  double zring[ZR][128];
  double z[1];             // [C][D], dynamic
};

__device__ __forceinline__ void cp_async8(void *dst, const void *src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(
                   static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
               "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Sum over the warp of one fp64 value per lane, the same on every lane (xor
// butterfly: partners add the same two operands, so all lanes agree bit for
// bit, and lane 0's order is that of a halving tree).
__device__ __forceinline__ double warp_sum(double s) {
#pragma unroll
  for (int off = 16; off; off >>= 1) s = __dadd_rn(s, __shfl_xor_sync(FULL, s, off));
  return s;
}

// Ward loss n_a n_b / (n_a + n_b) * |z_a / n_a - z_b / n_b|^2 (Chlience
// section 5.2, Corollary 1), means formed as z * (1 / n): within an ulp of
// z / n, so merge choices agree with the oracle whenever the best and second
// best losses differ by more than rounding.
template <int QD>
__device__ __forceinline__ double ward_loss(const EngSmem *sm, const double *z, int D, int sa,
                                            int sb, int lane) {
  const double na = (double)sm->n[sa], nb = (double)sm->n[sb];
  const double ia = sm->rn[sa], ib = sm->rn[sb];
  const double *za = z + (size_t)sa * D + lane, *zb = z + (size_t)sb * D + lane;
  double s = 0.0;
#pragma unroll
  for (int q = 0; q < QD; q++) {
    const double diff = __dsub_rn(__dmul_rn(za[32 * q], ia), __dmul_rn(zb[32 * q], ib));
    s = __dadd_rn(s, __dmul_rn(diff, diff));
  }
  const double f = __ddiv_rn(__dmul_rn(na, nb), __dadd_rn(na, nb));
  return __dmul_rn(f, warp_sum(s));
}

// Two independent Ward losses (a, b) and (b, c) in one pass (same arithmetic).
template <int QD>
__device__ __forceinline__ void ward_loss2(const EngSmem *sm, const double *z, int D, int sa,
                                           int sb, int sc, int lane, double &l_ab, double &l_bc) {
  const double na = (double)sm->n[sa], nb = (double)sm->n[sb], nc = (double)sm->n[sc];
  const double ia = sm->rn[sa], ib = sm->rn[sb], ic = sm->rn[sc];
  const double *za = z + (size_t)sa * D + lane, *zb = z + (size_t)sb * D + lane,
               *zc = z + (size_t)sc * D + lane;
  double s1 = 0.0, s2 = 0.0;
#pragma unroll
  for (int q = 0; q < QD; q++) {
    const double mb = __dmul_rn(zb[32 * q], ib);
    const double d1 = __dsub_rn(__dmul_rn(za[32 * q], ia), mb);
    const double d2 = __dsub_rn(mb, __dmul_rn(zc[32 * q], ic));
    s1 = __dadd_rn(s1, __dmul_rn(d1, d1));
    s2 = __dadd_rn(s2, __dmul_rn(d2, d2));
  }
#pragma unroll
  for (int off = 16; off; off >>= 1) {
    s1 = __dadd_rn(s1, __shfl_xor_sync(FULL, s1, off));
    s2 = __dadd_rn(s2, __shfl_xor_sync(FULL, s2, off));
  }
  const double f1 = __ddiv_rn(__dmul_rn(na, nb), __dadd_rn(na, nb));
  const double f2 = __ddiv_rn(__dmul_rn(nb, nc), __dadd_rn(nb, nc));
  l_ab = __dmul_rn(f1, s1);
  l_bc = __dmul_rn(f2, s2);
}

// Information density of the union of slots a and b (Chlience section 5.2):
// (I_a + I_b) / (n_a + n_b), the oracle's operation order.
__device__ __forceinline__ double info_density(const EngSmem *sm, int sa, int sb) {
  return __ddiv_rn(__dadd_rn(sm->info[sa], sm->info[sb]),
                   __dadd_rn((double)sm->n[sa], (double)sm->n[sb]));
}

// Leftmost argmin of loss[0 .. L-1] (L >= 1).  Losses are non-negative and
// finite, so their bit patterns order like their values: three 32-bit warp
// reductions (high word, low word, index) replace an fp64 shuffle tree.
__device__ __forceinline__ int argmin_leftmost(const double *loss, int L, int lane) {
  unsigned long long best = ~0ull;
  int bi = 0x7fffffff;
#pragma unroll
  for (int q = 0; q < 4; q++) {
    const int p = lane + 32 * q;
    if (p < L) {
      const unsigned long long key = (unsigned long long)__double_as_longlong(loss[p]);
      if (key < best) {
        best = key;
        bi = p;
      }
    }
  }
  const unsigned hi = __reduce_min_sync(FULL, (unsigned)(best >> 32));
  const unsigned lo = __reduce_min_sync(FULL, (unsigned)(best >> 32) == hi ? (unsigned)best : ~0u);
  const bool cand = best == (((unsigned long long)hi << 32) | lo);
  return (int)__reduce_min_sync(FULL, cand ? (unsigned)bi : 0x7fffffffu);
}

template <int D>
__global__ void __launch_bounds__(32) k_engine(Dims dm, Plan pl, CallArgs ca) {
  constexpr int QD = D / 32;
  extern __shared__ __align__(16) unsigned char eng_raw[];
  EngSmem *sm = reinterpret_cast<EngSmem *>(eng_raw);
  double *zs = sm->z;
  const int u = blockIdx.x, lane = threadIdx.x;
  const int C = dm.C, M = dm.M, W = dm.W, tiles = dm.tiles, amax = dm.amax, vmax = dm.vmax;
  const int opsmax = dm.opsmax, pmax = dm.pmax;
  const int Tw = tw_of(ca, u);
  int32_t *const dev_status = ca.dev_status;
  if (Tw == 0) {  // a ragged stream with no token in this window: nothing changes
    if (lane == 0) pl.nops[u] = 0;
    return;
  }
  // the head's cache
  int32_t *const c_order = ca.cache.order + (size_t)u * C;
  int64_t *const c_n = ca.cache.n + (size_t)u * C;
  int64_t *const c_ts = ca.cache.ts + (size_t)u * C;
  double *const c_loss = ca.cache.pair_loss + (size_t)u * C;
  double *const c_z = ca.cache.z + (size_t)u * C * D;
  // the head's plan
  const int nseg = pl.nseg[u];
  const int32_t *const ss = pl.seg_start + (size_t)u * (W + 1);
  const double *const zend = pl.z_end + (size_t)u * W * D;
  const double *const ztile_g = pl.z_tile + (size_t)u * tiles * D;
  int4 *const ops = pl.ops + (size_t)u * opsmax;
  int32_t *const tm0 = pl.tile_m0 + (size_t)u * tiles;
  int32_t *const tat = pl.tile_atoms + (size_t)u * tiles * amax;
  int32_t *const tnev = pl.tile_nev + (size_t)u * tiles;
  int32_t *const toff = pl.tile_ev_off + (size_t)u * tiles * M;
  int32_t *const tmrg = pl.tile_ev_mrg + (size_t)u * tiles * M;
  float *const ver_z = pl.ver_z + (size_t)u * vmax * D;
  float *const ver_n = pl.ver_n + (size_t)u * vmax;
  int32_t *const tr_t = ca.trace.merge_t ? ca.trace.merge_t + (size_t)u * ca.trace.cap : nullptr;
  int32_t *const tr_i = ca.trace.merge_i ? ca.trace.merge_i + (size_t)u * ca.trace.cap : nullptr;
  const bool tracing = ca.trace.merge_count != nullptr;
  const int tcap = ca.trace.cap;
  const bool info = dm.info != 0;
  double *const c_info = info ? ca.info_slot + (size_t)u * C : nullptr;
  const double *const seg_info = info ? pl.seg_info + (size_t)u * W : nullptr;

  // ---- segment-end sums: prefetch ring ------------------------------------
  auto zfetch = [&](int g) {
    if (g < nseg) {
      double *dst = sm->zring[g % ZR] + lane;
      const double *src = zend + (size_t)g * D + lane;
#pragma unroll
      for (int q = 0; q < QD; q++) cp_async8(dst + 32 * q, src + 32 * q);
    }
    cp_async_commit();
  };
#pragma unroll 1
  for (int g = 0; g < ZR; g++) zfetch(g);
  int zcons = 0;  // next z_end row to take (rows are taken in order)
  // z_end[zcons] -> dst (lane-owned dims); then refill its ring slot
  auto ztake = [&](double *dst) {
    cp_async_wait<ZR - 1>();
    const double *src = sm->zring[zcons % ZR] + lane;
#pragma unroll
    for (int q = 0; q < QD; q++) dst[lane + 32 * q] = src[32 * q];
    zfetch(zcons + ZR);
    zcons++;
  };

  // ---- load the head's summaries ------------------------------------------
  int m = ca.cache.m[u];
  const int64_t t0 = ca.cache.t[u];
  // the cosine / Ward policy does not continue a cache of the information
  // policy (its pair entries are densities, its prev_r an information score)
  if (!info && lane == 0 && c_loss[C - 1] < 0.0) set_status(dev_status, DLA_ERR_UNSUPPORTED);
  if (lane < 4) sm->used[lane] = 0u;
  __syncwarp();
  for (int p = lane; p < C; p += 32) {
    const int o = c_order[p];
    sm->order[p] = o;
    const long long nn = c_n[p];
    sm->n[p] = nn;
    sm->rn[p] = __drcp_rn((double)nn);
    sm->ts[p] = c_ts[p];
    sm->loss[p] = c_loss[p];
    sm->sver[p] = -1;
    sm->lastmod[p] = -1;
    sm->info[p] = info ? c_info[p] : 0.0;
    if (p < m) atomicOr(&sm->used[o >> 5], 1u << (o & 31));
  }
  for (int i = lane; i < C * D; i += 32) zs[i] = c_z[i];
  __syncwarp();
  // lane w < 4 keeps the used-slot bits of slots 32w .. 32w + 31
  uint32_t uw = lane < 4 ? sm->used[lane] : 0u;
  const uint32_t valid_bits = lane * 32 >= C ? 0u : (C - lane * 32 >= 32 ? ~0u : ((1u << (C - lane * 32)) - 1u));
  // lowest free slot
  auto alloc_slot = [&]() -> int {
    const uint32_t fr = ~uw & valid_bits;
    const unsigned bal = __ballot_sync(FULL, fr != 0u);
    if (bal == 0u) {
      if (lane == 0) set_status(dev_status, DLA_ERR_INVARIANT);
      return 0;
    }
    const int w = __ffs(bal) - 1;
    const int bit = __ffs(__shfl_sync(FULL, fr, w)) - 1;
    if (lane == w) uw |= 1u << bit;
    return w * 32 + bit;
  };

  int nops = 0, nver = 0;
  int ptile = -1, pk = 0;  // tile of the last piece and pieces emitted in it
  auto emit = [&](int op, int a, int b, int c) {
    if (lane == 0) {
      if (nops < opsmax) ops[nops] = make_int4(op, a, b, c);
      else set_status(dev_status, DLA_ERR_INVARIANT);
    }
    nops++;
  };
  // tokens [from, from + cnt) join the open state `slot`: a tensor-core piece
  // when long enough (and the path has pieces), else SIMT rank-1 adds
  auto emit_add = [&](int slot, int from, int cnt) {
    if (pmax > 0 && cnt >= PIECE_MIN) {
      const int tl = from / M;  // a run never crosses a tile boundary
      if (tl != ptile) {
        ptile = tl;
        pk = 0;
      }
      const int id = tl * PIECES_PER_TILE + pk++;
      if (id >= pmax && lane == 0) set_status(dev_status, DLA_ERR_INVARIANT);
      emit(OP_ADDP, slot, id, cnt);
    } else {
      emit(OP_ADD, slot, from, cnt);
    }
  };
  if (m > 0) emit(OP_LOAD, sm->order[m - 1], 0, 0);
  int mcount = tracing ? ca.trace.merge_count[u] : 0;
  const bool cont0 = nseg > 0 && pl.b[(size_t)u * W] == 0;  // token 0 continues the open state

  // segment starts, 32 per lane-register chunk, the next chunk in flight
  int sbase = 0;
  int ssA = lane < nseg ? ss[lane] : 0x7fffffff;
  int ssB = 32 + lane < nseg ? ss[32 + lane] : 0x7fffffff;

  int j = 0;
  int cur_from = 0;  // first window token not yet added to the open state
  double ztile[QD];  // open-state partial sum before the next tile
#pragma unroll
  for (int q = 0; q < QD; q++) ztile[q] = 0.0;
#pragma unroll 1
  for (int c = 0; c < tiles && c * M < Tw; c++) {
    const int T0 = c * M;
    const int Tend = min(T0 + M, Tw);
    double ztile_cur[QD];
#pragma unroll
    for (int q = 0; q < QD; q++) {
      ztile_cur[q] = ztile[q];
      ztile[q] = (c + 1 < tiles && (c + 1) * M < Tw) ? ztile_g[(size_t)(c + 1) * D + lane + 32 * q] : 0.0;
    }
    // ---- states present just before the tile ----------------------------
    if (m > 0 && T0 > cur_from) {
      const int os = sm->order[m - 1];
      emit_add(os, cur_from, T0 - cur_from);
      if (lane == 0) sm->n[os] += T0 - cur_from;
      cur_from = T0;
    }
    __syncwarp();
    const int m0 = m;
#pragma unroll 1
    for (int p0 = 0; p0 < m0; p0 += 32) {
      const int p = p0 + lane;
      const int slot = p < m0 ? sm->order[p] : 0;
      const int sv = p < m0 ? sm->sver[slot] : 0;
      const bool need = p < m0 && (p == m0 - 1 || sv < 0);
      // a sealed state whose value came from a STORE / MERGE of this window
      // gets its version id patched into that op; others get a SHADOW op
      const int lm = (need && p != m0 - 1) ? sm->lastmod[slot] : -1;
      const bool patch = lm >= 0;
      const unsigned bal = __ballot_sync(FULL, need);
      const unsigned bal_emit = __ballot_sync(FULL, need && !patch);
      const unsigned below = (1u << lane) - 1u;
      const int rank = __popc(bal & below);
      if (need) {
        const int v = nver + rank;
        if (patch) {
          if (lm < opsmax) ops[lm].w = v + 1;
          sm->lastmod[slot] = -1;
        } else {
          const int erank = __popc(bal_emit & below);
          if (nops + erank < opsmax) ops[nops + erank] = make_int4(OP_SHADOW, slot, v, 0);
          else set_status(dev_status, DLA_ERR_INVARIANT);
        }
        if (p != m0 - 1) sm->sver[slot] = v;
        tat[(size_t)c * amax + p] = v;
      } else if (p < m0) {
        tat[(size_t)c * amax + p] = sv;
      }
      // sums and counts of the new versions (lanes over dimensions)
      unsigned todo = bal;
      while (todo) {
        const int l = __ffs(todo) - 1;
        todo &= todo - 1;
        const int pv = p0 + l;
        const int sl = __shfl_sync(FULL, slot, l);
        const int v = nver + __popc(bal & ((1u << l) - 1u));
        float *zv = ver_z + (size_t)v * D + lane;
        if (pv == m0 - 1 && c > 0) {
#pragma unroll
          for (int q = 0; q < QD; q++) zv[32 * q] = (float)ztile_cur[q];
        } else {
          const double *zsrc = zs + (size_t)sl * D + lane;
#pragma unroll
          for (int q = 0; q < QD; q++) zv[32 * q] = (float)zsrc[32 * q];
        }
        if (lane == 0) ver_n[v] = (float)sm->n[sl];
      }
      nver += __popc(bal);
      nops += __popc(bal_emit);
      __syncwarp();
    }
    if (nver > vmax && lane == 0) set_status(dev_status, DLA_ERR_INVARIANT);
    if (lane == 0) tm0[c] = m0;
    // ---- boundaries inside the tile --------------------------------------
    int nev = 0;
#pragma unroll 1
    while (j < nseg) {
      if (j - sbase == 32) {
        sbase += 32;
        ssA = ssB;
        ssB = sbase + 32 + lane < nseg ? ss[sbase + 32 + lane] : 0x7fffffff;
      }
      const int s = __shfl_sync(FULL, ssA, j - sbase);
      if (s >= Tend) break;
      if (!(s == 0 && cont0)) {
        int mrg = EV_NO_MERGE;
        if (m > 0) {
          const int os = sm->order[m - 1];
          if (s > cur_from) {
            emit_add(os, cur_from, s - cur_from);
            if (lane == 0) sm->n[os] += s - cur_from;
          }
          if (j >= 1) ztake(zs + (size_t)os * D);
          if (info && j >= 1 && lane == 0) sm->info[os] = seg_info[j - 1];
          __syncwarp();
          // seal: the open state joins the sealed list (all m states sealed)
          if (lane == 0) sm->rn[os] = __drcp_rn((double)sm->n[os]);
          __syncwarp();
          if (m >= 2) {
            const double l = info ? info_density(sm, sm->order[m - 2], os)
                                  : ward_loss<QD>(sm, zs, D, sm->order[m - 2], os, lane);
            if (lane == 0) sm->loss[m - 2] = l;
          }
          __syncwarp();
          if (m == C) {
            const int is = argmin_leftmost(sm->loss, C - 1, lane);
            const int a = sm->order[is], bb = sm->order[is + 1];
            {
              double *za = zs + (size_t)a * D + lane;
              const double *zb = zs + (size_t)bb * D + lane;
#pragma unroll
              for (int q = 0; q < QD; q++) za[32 * q] = __dadd_rn(za[32 * q], zb[32 * q]);
            }
            if (bb == os) {
              // the just-sealed state is the right member: its registers go
              // straight into the left one, it is never stored
              if (lane == 0) sm->lastmod[a] = nops;
              emit(OP_MERGEO, a, 0, 0);
            } else {
              if (lane == 0) {
                sm->lastmod[os] = nops;
                sm->lastmod[a] = nops + 1;
              }
              emit(OP_STORE, os, 0, 0);
              emit(OP_MERGE, a, bb, 0);
            }
            if (lane == (bb >> 5)) uw &= ~(1u << (bb & 31));
            // drop position is + 1 from the order and pair is from the losses
            int32_t ov[4];
            double lv[4];
#pragma unroll
            for (int q = 0; q < 4; q++) {
              const int p = lane + 32 * q;
              ov[q] = (p >= is + 1 && p + 1 < C) ? sm->order[p + 1] : 0;
              lv[q] = (p >= is + 1 && p + 1 < C - 1) ? sm->loss[p + 1] : 0.0;
            }
            __syncwarp();
#pragma unroll
            for (int q = 0; q < 4; q++) {
              const int p = lane + 32 * q;
              if (p >= is + 1 && p + 1 < C) sm->order[p] = ov[q];
              if (p >= is + 1 && p + 1 < C - 1) sm->loss[p] = lv[q];
            }
            if (lane == 0) {
              const long long na = sm->n[a] + sm->n[bb];
              sm->n[a] = na;
              sm->rn[a] = __drcp_rn((double)na);
              if (info) sm->info[a] = __dadd_rn(sm->info[a], sm->info[bb]);
              sm->sver[a] = -1;
              sm->sver[bb] = -1;
            }
            __syncwarp();
            m -= 1;  // C - 1 sealed
            // the merged state's new neighbour losses
            const bool left = is >= 1, right = is + 1 <= m - 1;
            const int sl = sm->order[left ? is - 1 : is];
            const int sr = sm->order[right ? is + 1 : is];
            double l_left, l_right;
            if (info) {
              l_left = info_density(sm, sl, a);
              l_right = info_density(sm, a, sr);
            } else {
              ward_loss2<QD>(sm, zs, D, sl, a, sr, lane, l_left, l_right);
            }
            if (lane == 0) {
              if (left) sm->loss[is - 1] = l_left;
              if (right) sm->loss[is] = l_right;
            }
            __syncwarp();
            mrg = is;
            if (tracing) {
              if (mcount < tcap) {
                if (lane == 0) {
                  tr_t[mcount] = (int32_t)(t0 + s);
                  tr_i[mcount] = is;
                }
              } else if (lane == 0) {
                set_status(dev_status, DLA_ERR_TRACE_OVERFLOW);
              }
              mcount++;
            }
          } else {
            if (lane == 0) sm->lastmod[os] = nops;
            emit(OP_STORE, os, 0, 0);
          }
        }
        // open a new state at s
        const int slot = alloc_slot();
        emit(OP_ZERO, slot, 0, 0);
        {
          double *zn = zs + (size_t)slot * D + lane;
#pragma unroll
          for (int q = 0; q < QD; q++) zn[32 * q] = 0.0;
        }
        if (lane == 0) {
          sm->n[slot] = 0;
          sm->ts[slot] = t0 + s;
          sm->info[slot] = 0.0;
          sm->order[m] = slot;
          sm->sver[slot] = -1;
          sm->lastmod[slot] = -1;
          toff[(size_t)c * M + nev] = s - T0;
          tmrg[(size_t)c * M + nev] = mrg;
        }
        __syncwarp();
        m += 1;
        cur_from = s;
        nev++;
      }
      j++;
    }
    if (lane == 0) tnev[c] = nev;
  }
  // ---- window end -------------------------------------------------------
  if (m > 0) {
    const int os = sm->order[m - 1];
    if (Tw > cur_from) {
      emit_add(os, cur_from, Tw - cur_from);
      if (lane == 0) sm->n[os] += Tw - cur_from;
    }
    emit(OP_STORE, os, 0, 0);
    if (nseg >= 1) ztake(zs + (size_t)os * D);
    if (info && nseg >= 1 && lane == 0) sm->info[os] = seg_info[nseg - 1];
  }
  cp_async_wait<0>();
  __syncwarp();
  for (int p = lane; p < C; p += 32) {
    c_order[p] = sm->order[p];
    c_n[p] = sm->n[p];
    c_ts[p] = sm->ts[p];
    // pair_loss[C - 1] belongs to no pair: under the information policy it
    // marks the cache as holding that policy's states (CACHE_INFO_MARK)
    c_loss[p] = (info && p == C - 1) ? CACHE_INFO_MARK : sm->loss[p];
    if (info) c_info[p] = sm->info[p];
  }
  for (int i = lane; i < C * D; i += 32) c_z[i] = zs[i];
  if (lane == 0) {
    ca.cache.m[u] = m;
    ca.cache.t[u] = t0 + Tw;
    ca.cache.prev_r[u] = pl.r[(size_t)u * W + Tw - 1];
    pl.nops[u] = min(nops, opsmax);
    if (tracing) ca.trace.merge_count[u] = mcount;
  }
  const size_t krow = ((size_t)u * dm.T + ca.w0 + Tw - 1) * D;
  for (int d2 = lane; d2 < D; d2 += 32) ca.cache.prev_k[(size_t)u * D + d2] = load_in(ca.k, ca.in_dtype, krow + d2);
}

// ------------------------------------------------------ unbounded engine ----
// The unbounded policy, DLA(I) (the ablation row "Mamba-2 + DLA(I)" of the
// Chlience page's ablation table): the same walk over tiles and segment
// starts, with no capacity merge.  Every segment stays a state of its own, so
// a sealed state never changes again: its version is written once, and its
// fp64 z goes straight to the cache when it is sealed.  The cache's C slots
// are storage only; a stream that needs more states than C sets
// DLA_ERR_CAPACITY (its later boundaries are then not opened and its results
// are unspecified).  Per-slot summaries (time order, version, last op, n, ts)
// sit in shared memory for up to DLA_MAX_SLOTS slots; lane w keeps the
// used-slot bits of slots 32w .. 32w + 31.
template <int D>
__global__ void __launch_bounds__(32) k_engine_unb(Dims dm, Plan pl, CallArgs ca) {
  constexpr int QD = D / 32;
  extern __shared__ __align__(16) unsigned char unb_raw[];
  const int C = dm.C, M = dm.M, W = dm.W, tiles = dm.tiles, amax = dm.amax, vmax = dm.vmax;
  const int opsmax = dm.opsmax, pmax = dm.pmax;
  double(*zring)[128] = reinterpret_cast<double(*)[128]>(unb_raw);
  double *zdump = reinterpret_cast<double *>(unb_raw + sizeof(double) * ZR * 128);
  long long *s_n = reinterpret_cast<long long *>(zdump + 128);
  long long *s_ts = s_n + C;
  int32_t *s_order = reinterpret_cast<int32_t *>(s_ts + C);
  int32_t *s_sver = s_order + C;
  int32_t *s_lastmod = s_sver + C;
  const int u = blockIdx.x, lane = threadIdx.x;
  const int Tw = tw_of(ca, u);
  int32_t *const dev_status = ca.dev_status;
  if (Tw == 0) {  // a ragged stream with no token in this window: nothing changes
    if (lane == 0) pl.nops[u] = 0;
    return;
  }
  int32_t *const c_order = ca.cache.order + (size_t)u * C;
  int64_t *const c_n = ca.cache.n + (size_t)u * C;
  int64_t *const c_ts = ca.cache.ts + (size_t)u * C;
  double *const c_loss = ca.cache.pair_loss + (size_t)u * C;
  double *const c_z = ca.cache.z + (size_t)u * C * D;
  const int nseg = pl.nseg[u];
  const int32_t *const ss = pl.seg_start + (size_t)u * (W + 1);
  const double *const zend = pl.z_end + (size_t)u * W * D;
  const double *const ztile_g = pl.z_tile + (size_t)u * tiles * D;
  int4 *const ops = pl.ops + (size_t)u * opsmax;
  int32_t *const tm0 = pl.tile_m0 + (size_t)u * tiles;
  int32_t *const tat = pl.tile_atoms + (size_t)u * tiles * amax;
  int32_t *const tnev = pl.tile_nev + (size_t)u * tiles;
  int32_t *const toff = pl.tile_ev_off + (size_t)u * tiles * M;
  int32_t *const tmrg = pl.tile_ev_mrg + (size_t)u * tiles * M;
  float *const ver_z = pl.ver_z + (size_t)u * vmax * D;
  float *const ver_n = pl.ver_n + (size_t)u * vmax;

  // only an empty cache or one of this policy is continued
  if (lane == 0 && ca.cache.t[u] > 0 && c_loss[C - 1] != CACHE_UNBOUNDED_MARK)
    set_status(dev_status, DLA_ERR_UNSUPPORTED);

  // ---- segment-end sums: prefetch ring (as in k_engine) ----------------------
  auto zfetch = [&](int g) {
    if (g < nseg) {
      double *dst = zring[g % ZR] + lane;
      const double *src = zend + (size_t)g * D + lane;
#pragma unroll
      for (int q = 0; q < QD; q++) cp_async8(dst + 32 * q, src + 32 * q);
    }
    cp_async_commit();
  };
#pragma unroll 1
  for (int g = 0; g < ZR; g++) zfetch(g);
  int zcons = 0;
  auto ztake = [&](double *dst) {
    cp_async_wait<ZR - 1>();
    const double *src = zring[zcons % ZR] + lane;
#pragma unroll
    for (int q = 0; q < QD; q++) dst[lane + 32 * q] = src[32 * q];
    zfetch(zcons + ZR);
    zcons++;
  };

  int m = ca.cache.m[u];
  const int64_t t0 = ca.cache.t[u];
  uint32_t uw = 0u;  // this lane's word of the used-slot bits
  for (int p = lane; p < C; p += 32) {
    s_order[p] = c_order[p];
    s_n[p] = c_n[p];
    s_ts[p] = c_ts[p];
    s_sver[p] = -1;
    s_lastmod[p] = -1;
  }
  __syncwarp();
  for (int p = 0; p < m; p++) {
    const int o = s_order[p];
    if (lane == (o >> 5)) uw |= 1u << (o & 31);
  }
  const uint32_t valid_bits =
      lane * 32 >= C ? 0u : (C - lane * 32 >= 32 ? ~0u : ((1u << (C - lane * 32)) - 1u));
  auto alloc_slot = [&]() -> int {
    const uint32_t fr = ~uw & valid_bits;
    const unsigned bal = __ballot_sync(FULL, fr != 0u);
    if (bal == 0u) {  // m < C with no free slot: an inconsistent cache
      if (lane == 0) set_status(dev_status, DLA_ERR_INVARIANT);
      return 0;
    }
    const int w = __ffs(bal) - 1;
    const int bit = __ffs(__shfl_sync(FULL, fr, w)) - 1;
    if (lane == w) uw |= 1u << bit;
    return w * 32 + bit;
  };

  int nops = 0, nver = 0;
  int ptile = -1, pk = 0;
  auto emit = [&](int op, int a, int b, int c) {
    if (lane == 0) {
      if (nops < opsmax) ops[nops] = make_int4(op, a, b, c);
      else set_status(dev_status, DLA_ERR_INVARIANT);
    }
    nops++;
  };
  auto emit_add = [&](int slot, int from, int cnt) {
    if (pmax > 0 && cnt >= PIECE_MIN) {
      const int tl = from / M;
      if (tl != ptile) {
        ptile = tl;
        pk = 0;
      }
      const int id = tl * PIECES_PER_TILE + pk++;
      if (id >= pmax && lane == 0) set_status(dev_status, DLA_ERR_INVARIANT);
      emit(OP_ADDP, slot, id, cnt);
    } else {
      emit(OP_ADD, slot, from, cnt);
    }
  };
  if (m > 0) emit(OP_LOAD, s_order[m - 1], 0, 0);
  const bool cont0 = nseg > 0 && pl.b[(size_t)u * W] == 0;
  int sbase = 0;
  int ssA = lane < nseg ? ss[lane] : 0x7fffffff;
  int ssB = 32 + lane < nseg ? ss[32 + lane] : 0x7fffffff;
  int j = 0;
  int cur_from = 0;
  double ztile[QD];
#pragma unroll
  for (int q = 0; q < QD; q++) ztile[q] = 0.0;
#pragma unroll 1
  for (int c = 0; c < tiles && c * M < Tw; c++) {
    const int T0 = c * M;
    const int Tend = min(T0 + M, Tw);
    double ztile_cur[QD];
#pragma unroll
    for (int q = 0; q < QD; q++) {
      ztile_cur[q] = ztile[q];
      ztile[q] = (c + 1 < tiles && (c + 1) * M < Tw) ? ztile_g[(size_t)(c + 1) * D + lane + 32 * q] : 0.0;
    }
    if (m > 0 && T0 > cur_from) {
      const int os = s_order[m - 1];
      emit_add(os, cur_from, T0 - cur_from);
      if (lane == 0) s_n[os] += T0 - cur_from;
      cur_from = T0;
    }
    __syncwarp();
    // ---- the states present before the tile: every live state --------------
    const int m0 = m;
#pragma unroll 1
    for (int p0 = 0; p0 < m0; p0 += 32) {
      const int p = p0 + lane;
      const int slot = p < m0 ? s_order[p] : 0;
      const int sv = p < m0 ? s_sver[slot] : 0;
      const bool need = p < m0 && (p == m0 - 1 || sv < 0);
      const int lm = (need && p != m0 - 1) ? s_lastmod[slot] : -1;
      const bool patch = lm >= 0;
      const unsigned bal = __ballot_sync(FULL, need);
      const unsigned bal_emit = __ballot_sync(FULL, need && !patch);
      const unsigned below = (1u << lane) - 1u;
      const int rank = __popc(bal & below);
      if (need) {
        const int v = nver + rank;
        if (patch) {
          if (lm < opsmax) ops[lm].w = v + 1;
          s_lastmod[slot] = -1;
        } else {
          const int erank = __popc(bal_emit & below);
          if (nops + erank < opsmax) ops[nops + erank] = make_int4(OP_SHADOW, slot, v, 0);
          else set_status(dev_status, DLA_ERR_INVARIANT);
        }
        if (p != m0 - 1) s_sver[slot] = v;
        tat[(size_t)c * amax + p] = min(v, vmax - 1);  // (v >= vmax is flagged below)
      } else if (p < m0) {
        tat[(size_t)c * amax + p] = sv;
      }
      unsigned todo = bal;
      while (todo) {
        const int l = __ffs(todo) - 1;
        todo &= todo - 1;
        const int pv = p0 + l;
        const int sl = __shfl_sync(FULL, slot, l);
        const int v = nver + __popc(bal & ((1u << l) - 1u));
        if (v < vmax) {
          float *zv = ver_z + (size_t)v * D + lane;
          if (pv == m0 - 1 && c > 0) {
#pragma unroll
            for (int q = 0; q < QD; q++) zv[32 * q] = (float)ztile_cur[q];
          } else {
            const double *zsrc = c_z + (size_t)sl * D + lane;
#pragma unroll
            for (int q = 0; q < QD; q++) zv[32 * q] = (float)zsrc[32 * q];
          }
          if (lane == 0) ver_n[v] = (float)s_n[sl];
        }
      }
      nver += __popc(bal);
      nops += __popc(bal_emit);
      __syncwarp();
    }
    if (nver > vmax && lane == 0) set_status(dev_status, DLA_ERR_INVARIANT);
    if (lane == 0) tm0[c] = m0;
    // ---- boundaries inside the tile ----------------------------------------
    int nev = 0;
#pragma unroll 1
    while (j < nseg) {
      if (j - sbase == 32) {
        sbase += 32;
        ssA = ssB;
        ssB = sbase + 32 + lane < nseg ? ss[sbase + 32 + lane] : 0x7fffffff;
      }
      const int s = __shfl_sync(FULL, ssA, j - sbase);
      if (s >= Tend) break;
      if (!(s == 0 && cont0)) {
        if (m == C) {
          // no slot left for a new state: report it; the token stays in the
          // open state (the ring entry of the segment is consumed)
          if (lane == 0) set_status(dev_status, DLA_ERR_CAPACITY);
          if (j >= 1) ztake(zdump);
          j++;
          continue;
        }
        if (m > 0) {
          const int os = s_order[m - 1];
          if (s > cur_from) {
            emit_add(os, cur_from, s - cur_from);
            if (lane == 0) s_n[os] += s - cur_from;
          }
          if (j >= 1) ztake(c_z + (size_t)os * D);  // the sealed state's final z
          if (lane == 0) s_lastmod[os] = nops;
          emit(OP_STORE, os, 0, 0);
        }
        const int slot = alloc_slot();
        emit(OP_ZERO, slot, 0, 0);
        if (lane == 0) {
          s_n[slot] = 0;
          s_ts[slot] = t0 + s;
          s_order[m] = slot;
          s_sver[slot] = -1;
          s_lastmod[slot] = -1;
          toff[(size_t)c * M + nev] = s - T0;
          tmrg[(size_t)c * M + nev] = EV_NO_MERGE;
        }
        __syncwarp();
        m += 1;
        cur_from = s;
        nev++;
      }
      j++;
    }
    if (lane == 0) tnev[c] = nev;
  }
  // ---- window end ----------------------------------------------------------
  if (m > 0) {
    const int os = s_order[m - 1];
    if (Tw > cur_from) {
      emit_add(os, cur_from, Tw - cur_from);
      if (lane == 0) s_n[os] += Tw - cur_from;
    }
    emit(OP_STORE, os, 0, 0);
    if (nseg >= 1 && zcons < nseg) ztake(c_z + (size_t)os * D);
  }
  cp_async_wait<0>();
  __syncwarp();
  for (int p = lane; p < C; p += 32) {
    c_order[p] = s_order[p];
    c_n[p] = s_n[p];
    c_ts[p] = s_ts[p];
  }
  if (lane == 0) {
    c_loss[C - 1] = CACHE_UNBOUNDED_MARK;
    ca.cache.m[u] = m;
    ca.cache.t[u] = t0 + Tw;
    ca.cache.prev_r[u] = pl.r[(size_t)u * W + Tw - 1];
    pl.nops[u] = min(nops, opsmax);
  }
  const size_t krow = ((size_t)u * dm.T + ca.w0 + Tw - 1) * D;
  for (int d2 = lane; d2 < D; d2 += 32) ca.cache.prev_k[(size_t)u * D + d2] = load_in(ca.k, ca.in_dtype, krow + d2);
}

}  // namespace

// The score kernel also forms the tile sums for bf16 keys with tiles of
// SCORE_TOK rows; k_segsum then only combines them.
bool sums_in_score(const Dims &dm, const CallArgs &ca, int policy) {
  return ca.in_dtype == DLA_BF16 && dm.M == SCORE_TOK && policy == DLA_POLICY_DYNAMIC;
}

cudaError_t launch_score(const Dims &dm, const Plan &pl, const CallArgs &ca, int policy,
                         cudaStream_t s) {
  const bool bf = ca.in_dtype == DLA_BF16;
  const int sums = sums_in_score(dm, ca, policy) ? 1 : 0;
  if (sums) k_phi_table<<<(PHI_TAB + 255) / 256, 256, 0, s>>>(pl.phi_tab);
  const size_t sb = sizeof(uint32_t) * (SCORE_TOK + 2) * ((bf ? dm.D / 2 : dm.D) + 1);
  dim3 g((ca.Tw + SCORE_TOK - 1) / SCORE_TOK, dm.heads);
  if (bf) {
    cudaError_t e = cudaFuncSetAttribute(k_score<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sb);
    if (e != cudaSuccess) return e;
    k_score<true><<<g, SCORE_TOK, sb, s>>>(dm, pl, ca, policy, sums);
  } else {
    cudaError_t e = cudaFuncSetAttribute(k_score<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sb);
    if (e != cudaSuccess) return e;
    k_score<false><<<g, SCORE_TOK, sb, s>>>(dm, pl, ca, policy, 0);
  }
  return cudaGetLastError();
}

cudaError_t launch_segscan(const Dims &dm, const Plan &pl, const CallArgs &ca, cudaStream_t s) {
  k_segscan<<<dm.heads, 1024, 0, s>>>(dm, pl, ca);
  return cudaGetLastError();
}

cudaError_t launch_segsum(const Dims &dm, const Plan &pl, const CallArgs &ca, cudaStream_t s) {
  const dim3 g(dm.tiles, dm.heads);
  if (!dm.info && sums_in_score(dm, ca, DLA_POLICY_DYNAMIC)) {
    // the tile sums came with the score
  } else {
    k_tilesum_any<<<g, dm.D, 0, s>>>(dm, pl, ca);
  }
  k_segcombine<<<dim3(64, dm.heads), dm.D, 0, s>>>(dm, pl, ca);
  return cudaGetLastError();
}

// The engine is one latency-bound warp per head.  When every head gets an SM
// of its own, its CTA reserves most of that SM's shared memory, so the
// builder and phi kernels that run beside it take other SMs instead of
// competing for its issue slots (with more heads than SMs it keeps its own
// size, so that several engines share an SM rather than queue).
constexpr size_t ENGINE_SM_RESERVE = 200 * 1024;

static int sm_count() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      n = 1;
  }
  return n;
}

template <int D>
static cudaError_t launch_engine_d(const Dims &dm, const Plan &pl, const CallArgs &ca, cudaStream_t s) {
  size_t sb = sizeof(EngSmem) + sizeof(double) * ((size_t)dm.C * D - 1);
  if (dm.heads <= sm_count() && sb < ENGINE_SM_RESERVE) sb = ENGINE_SM_RESERVE;
  cudaError_t e = cudaFuncSetAttribute(k_engine<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sb);
  if (e != cudaSuccess) return e;
  k_engine<D><<<dm.heads, 32, sb, s>>>(dm, pl, ca);
  return cudaGetLastError();
}

template <int D>
static cudaError_t launch_engine_unb_d(const Dims &dm, const Plan &pl, const CallArgs &ca,
                                       cudaStream_t s) {
  size_t sb = sizeof(double) * (ZR * 128 + 128) + (size_t)dm.C * (2 * sizeof(long long) + 3 * sizeof(int32_t));
  if (dm.heads <= sm_count() && sb < ENGINE_SM_RESERVE) sb = ENGINE_SM_RESERVE;
  cudaError_t e = cudaFuncSetAttribute(k_engine_unb<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sb);
  if (e != cudaSuccess) return e;
  k_engine_unb<D><<<dm.heads, 32, sb, s>>>(dm, pl, ca);
  return cudaGetLastError();
}

cudaError_t launch_engine(const Dims &dm, const Plan &pl, const CallArgs &ca, cudaStream_t s) {
  if (dm.unb) {
    switch (dm.D) {
      case 32: return launch_engine_unb_d<32>(dm, pl, ca, s);
      case 64: return launch_engine_unb_d<64>(dm, pl, ca, s);
      case 128: return launch_engine_unb_d<128>(dm, pl, ca, s);
    }
    return cudaErrorInvalidValue;
  }
  switch (dm.D) {
    case 32: return launch_engine_d<32>(dm, pl, ca, s);
    case 64: return launch_engine_d<64>(dm, pl, ca, s);
    case 128: return launch_engine_d<128>(dm, pl, ca, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace dla
