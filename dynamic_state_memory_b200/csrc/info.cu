// info.cu -- score kernel of the information policy (Dynamic Linear
// Attention | Chlience Paper Archive, section 5.1).  Token t's state
// s_t = v_t u_t^T (u = phi(k)) is compared with the open state S:
//   I_t = |N(s_t) - N(S)|_F / (|N(S)|_F + eps),  N(X) = X / sqrt(|X|^2 / (d_k d_v) + eps),
// with eps = 1e-6; b_t = [I_t >= tau], and the first token of a stream opens
// a state with I = 0.
//
// A cluster of two CTAs of 2D threads per head walks the window in blocks of
// INFO_K tokens.  CTA r of the pair keeps rows r D/2 .. + D/2 of S in fp64
// registers: thread i holds row r D/2 + i % (D/2), columns (i / (D/2)) D/4
// .. + D/4.  Each warp's partial sums of the block's inner products go to
// both CTAs' shared memory (distributed shared memory), one cluster barrier
// later both CTAs add them in the same order and take the same decisions;
// rank 0 alone writes the outputs.  Writing x_t = <s_t, S> = v_t^T S u_t,
//   |N(s) - N(S)|^2 = |s|^2 / ra + |S|^2 / rb - 2 x_t / sqrt(ra rb)
// (ra, rb: the two squared RMS denominators; with g = 1 / sqrt(rb) the
// middle term is |S|^2 g^2 and |N(S)| = |S| g), so a block needs per token
// v_t^T S0 u_t against the state S0 at the block's start (one pass over the
// registers with INFO_K accumulators and one block reduction) and the Gram
// terms (v_t . v_j)(u_t . u_j) of the block's earlier tokens j (staged per
// chunk).  The block's decisions then follow in token order from scalars:
// a token after an in-block boundary at jb sees x_t = sum_{j=jb}^{t-1} of its
// Gram terms, and |S|^2 follows |S + s|^2 = |S|^2 + 2x + |s|^2.  A second
// pass adds the block's tokens from its last boundary on to the registers.
// The order of the fp64 sums differs from an elementwise evaluation, so the
// scores agree with one to rounding (about 1e-7 absolute where I is near 0,
// far less elsewhere) and the decisions wherever |I_t - tau| exceeds that.
//
// Outputs per window: the scores r, the boundary flags b (and the trace's),
// and seg_info[j], the open state's score sum at the end of window piece j
// (pieces as numbered by the segment scan: piece 0 starts at the window's
// first token, piece j > 0 at the j-th later boundary).  S, |S|^2, the open
// state's score sum and the has-open flag carry to the call's next window.
#include <cooperative_groups.h>

#include "dla_internal.cuh"

namespace cg = cooperative_groups;

namespace dla {
namespace {

constexpr unsigned FULL = 0xffffffffu;
constexpr int INFO_K = 8;       // tokens decided per pass over the state
constexpr int INFO_CHUNK = 32;  // tokens staged per chunk (a multiple of INFO_K)
constexpr double INFO_EPS = 1e-6;

template <int D>
struct InfoSmem {
  uint32_t raw[2][2][INFO_CHUNK * D];  // [buffer][k, v] input rows (room for fp32)
  double u[INFO_CHUNK][D];             // phi(k) in fp64
  double v[INFO_CHUNK][D];
  // per token: |s|^2, |s|^2 / ra and 1 / sqrt(ra), ra = |s|^2 / (d_k d_v) + eps
  double ss[INFO_CHUNK], ssra[INFO_CHUNK], rsa[INFO_CHUNK];
  double H[INFO_CHUNK][INFO_K];           // (v_t . v_j)(u_t . u_j), j an earlier token of t's block
  double red[2][INFO_K][2 * (2 * D / 32)];  // per-warp partials of both CTAs, by block parity
  int jb;                                 // the block's last boundary (-1: none)
};

__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                   static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
               "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_wait1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }

__device__ __forceinline__ double warp_sum(double s) {
#pragma unroll
  for (int off = 16; off; off >>= 1) s += __shfl_xor_sync(FULL, s, off);
  return s;
}

// Rows t0 .. t0 + INFO_CHUNK - 1 (window-local) of k and v into raw[buf];
// rows past the window are zero-filled instead of loaded.
template <int D>
__device__ void info_stage(InfoSmem<D> &sm, int buf, const Dims &dm, const CallArgs &ca, int u,
                           int t0, int esize, int Tw) {
  const int nrow = min(INFO_CHUNK, Tw - t0);
  const int rowbytes = D * esize;
  const int n16 = INFO_CHUNK * rowbytes / 16;
  for (int which = 0; which < 2; which++) {
    const char *src = static_cast<const char *>(which ? ca.v : ca.k) +
                      ((size_t)u * dm.T + ca.w0 + t0) * rowbytes;
    char *dst = reinterpret_cast<char *>(sm.raw[buf][which]);
    for (int e = threadIdx.x; e < n16; e += blockDim.x) {
      if ((e * 16) / rowbytes < nrow) cp_async16(dst + e * 16, src + (size_t)e * 16);
      else *reinterpret_cast<uint4 *>(dst + e * 16) = make_uint4(0, 0, 0, 0);
    }
  }
  cp_commit();
}

// raw[buf] -> u = phi(k), v in fp64; then each token's norm terms and the
// in-block Gram terms of the chunk.  Two barriers inside.
template <int D>
__device__ void info_prepare(InfoSmem<D> &sm, int buf, bool bf16) {
  for (int e = threadIdx.x; e < INFO_CHUNK * D; e += blockDim.x) {
    const int r = e / D, c = e % D;
    float kf, vf;
    if (bf16) {
      const uint16_t *kr = reinterpret_cast<const uint16_t *>(sm.raw[buf][0]);
      const uint16_t *vr = reinterpret_cast<const uint16_t *>(sm.raw[buf][1]);
      kf = __uint_as_float((uint32_t)kr[e] << 16);
      vf = __uint_as_float((uint32_t)vr[e] << 16);
    } else {
      kf = __uint_as_float(sm.raw[buf][0][e]);
      vf = __uint_as_float(sm.raw[buf][1][e]);
    }
    sm.u[r][c] = phi64((double)kf);
    sm.v[r][c] = (double)vf;
  }
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  for (int r = warp; r < INFO_CHUNK; r += nw) {
    double a = 0.0, b = 0.0;
    for (int c = lane; c < D; c += 32) {
      a = fma(sm.u[r][c], sm.u[r][c], a);
      b = fma(sm.v[r][c], sm.v[r][c], b);
    }
    a = warp_sum(a);
    b = warp_sum(b);
    if (lane == 0) {
      const double ss = a * b;  // |s_t|^2 = |v_t|^2 |u_t|^2
      const double ra = fma(ss, 1.0 / (double)(D * D), INFO_EPS);
      sm.ss[r] = ss;
      sm.ssra[r] = ss / ra;
      sm.rsa[r] = rsqrt(ra);
    }
  }
  // one thread per (token, earlier token of its block); each lane starts at
  // its own column so that the rows' equal-bank columns are not read at once
  for (int p = threadIdx.x; p < INFO_CHUNK * INFO_K; p += blockDim.x) {
    const int r = p / INFO_K, j = p % INFO_K;
    const int q = r - r % INFO_K + j;
    double h = 0.0;
    if (q < r) {
      double gv0 = 0.0, gv1 = 0.0, gu0 = 0.0, gu1 = 0.0;
      for (int cc = 0; cc < D; cc += 2) {
        const int c = (cc + 2 * lane) & (D - 1);
        gv0 = fma(sm.v[r][c], sm.v[q][c], gv0);
        gv1 = fma(sm.v[r][c + 1], sm.v[q][c + 1], gv1);
        gu0 = fma(sm.u[r][c], sm.u[q][c], gu0);
        gu1 = fma(sm.u[r][c + 1], sm.u[q][c + 1], gu1);
      }
      h = (gv0 + gv1) * (gu0 + gu1);
    }
    sm.H[r][j] = h;
  }
  __syncthreads();
}

template <int D>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(2 * D, 1)
    k_info_score(Dims dm, Plan pl, CallArgs ca) {
  constexpr int NT = 2 * D, HR = D / 2, EPT = D / 4, NW = NT / 32;
  extern __shared__ __align__(16) unsigned char info_raw[];
  InfoSmem<D> &sm = *reinterpret_cast<InfoSmem<D> *>(info_raw);
  cg::cluster_group cl = cg::this_cluster();
  const int rank = (int)cl.block_rank();
  const int u = blockIdx.x / 2, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // the lanes of a warp hold consecutive rows of one column quarter (for
  // D >= 64), so they read the same element of u: one broadcast per load
  const int a = rank * HR + tid % HR, c0 = (tid / HR) * EPT;
  // this warp's partials go to slot rank * NW + warp of both CTAs
  double(*const red_peer)[INFO_K][2 * NW] = cl.map_shared_rank(sm.red, rank ^ 1);
  const bool bf16 = ca.in_dtype == DLA_BF16;
  const int esize = bf16 ? 2 : 4;
  const double tau = (double)ca.tau;
  const double inv_d2 = 1.0 / (double)(D * D);  // a power of two: exact
  double *const carry = ca.info_S + (size_t)u * D * D + (size_t)rank * HR * D;
  double *const aux = ca.info_aux + (size_t)u * 4;
  double S[EPT];
  double sS, iopen;
  bool has_open;
  if (ca.w0 == 0) {
    // the decisions need the open state in fp64, which a cache does not
    // hold: this policy starts every stream from an empty cache
    if (rank == 0 && tid == 0 && (ca.cache.t[u] != 0 || ca.cache.m[u] != 0))
      set_status(ca.dev_status, DLA_ERR_UNSUPPORTED);
#pragma unroll
    for (int j = 0; j < EPT; j++) S[j] = 0.0;
    sS = 0.0;
    iopen = 0.0;
    has_open = false;
  } else {
#pragma unroll
    for (int j = 0; j < EPT; j++) S[j] = carry[(size_t)j * NT + tid];
    sS = aux[0];
    iopen = aux[1];
    has_open = aux[2] != 0.0;
  }
  double *const r_out = pl.r + (size_t)u * dm.W;
  uint8_t *const b_out = pl.b + (size_t)u * dm.W;
  uint8_t *const tr_b = ca.trace.boundary ? ca.trace.boundary + (size_t)u * dm.T + ca.w0 : nullptr;
  double *const seg = pl.seg_info + (size_t)u * dm.W;
  int sg = 0;  // current window piece
  const int Tw = tw_of(ca, u);
  const int nchunk = (Tw + INFO_CHUNK - 1) / INFO_CHUNK;
  info_stage<D>(sm, 0, dm, ca, u, 0, esize, Tw);
  int blk = 0;
#pragma unroll 1
  for (int ch = 0; ch < nchunk; ch++) {
    const int t0 = ch * INFO_CHUNK;
    __syncthreads();  // the previous chunk's passes are done with u, v, H
    if (ch + 1 < nchunk) info_stage<D>(sm, (ch + 1) & 1, dm, ca, u, t0 + INFO_CHUNK, esize, Tw);
    else cp_commit();  // an empty group keeps the wait count uniform
    cp_wait1();
    __syncthreads();
    info_prepare<D>(sm, ch & 1, bf16);
    const int nrow = min(INFO_CHUNK, Tw - t0);
#pragma unroll 1
    for (int r0 = 0; r0 < nrow; r0 += INFO_K, blk++) {
      const int nb = min(INFO_K, nrow - r0);
      // v_t^T S0 u_t for the block's tokens (rows past the window read the
      // zero-filled staging and are never used)
      double acc[INFO_K];
#pragma unroll
      for (int i = 0; i < INFO_K; i++) acc[i] = 0.0;
#pragma unroll
      for (int j = 0; j < EPT; j += 2) {
#pragma unroll
        for (int i = 0; i < INFO_K; i++) {
          const double2 w = *reinterpret_cast<const double2 *>(&sm.u[r0 + i][c0 + j]);
          acc[i] = fma(S[j], w.x, acc[i]);
          acc[i] = fma(S[j + 1], w.y, acc[i]);
        }
      }
      const int rb = blk & 1;
#pragma unroll
      for (int i = 0; i < INFO_K; i++) {
        const double p = warp_sum(sm.v[r0 + i][a] * acc[i]);
        if (lane == 0) {
          sm.red[rb][i][rank * NW + warp] = p;
          red_peer[rb][i][rank * NW + warp] = p;
        }
      }
      // both CTAs' partials of this block are in place (the peer can be at
      // most one block ahead, so the other parity is never overwritten early)
      cl.sync();
      // the block's decisions in token order, by warp 0 (its lanes agree);
      // the other warps wait: the fp64 pipe is the kernel's bound, so they
      // do not repeat this sequence
      if (warp == 0) {
        double A[INFO_K];
#pragma unroll
        for (int i = 0; i < INFO_K; i++) {
          double s = 0.0;
#pragma unroll
          for (int w = 0; w < 2 * NW; w++) s += sm.red[rb][i][w];
          A[i] = s;
        }
        int jb = -1;  // the block's last boundary so far
#pragma unroll
        for (int i = 0; i < INFO_K; i++) {
          if (i < nb) {
            const int t = t0 + r0 + i;
            double I = 0.0, x = 0.0;
            bool bnd = true;
            if (has_open) {
              x = jb < 0 ? A[i] : 0.0;
              for (int j = jb < 0 ? 0 : jb; j < i; j++) x += sm.H[r0 + i][j];
              // |N(s) - N(S)|^2 = |s|^2/ra + |S|^2 g^2 - 2 x g / sqrt(ra),
              // g = 1 / sqrt(|S|^2 / (d_k d_v) + eps); |N(S)| = |S| g
              const double g = rsqrt(fma(sS, inv_d2, INFO_EPS));
              const double num2 = fmax(sm.ssra[r0 + i] + sS * g * g - 2.0 * x * sm.rsa[r0 + i] * g, 0.0);
              I = sqrt(num2) / (sqrt(sS) * g + INFO_EPS);
              bnd = !(I < tau);
            }
            if (lane == 0 && rank == 0) {
              r_out[t] = I;
              b_out[t] = bnd ? 1 : 0;
              if (tr_b) tr_b[t] = bnd ? 1 : 0;
            }
            const double ssv = sm.ss[r0 + i];
            if (bnd) {
              if (t > 0) {
                if (lane == 0 && rank == 0) seg[sg] = iopen;
                sg++;
              }
              jb = i;
              sS = ssv;
              iopen = I;
              has_open = true;
            } else {
              sS = sS + 2.0 * x + ssv;
              iopen = iopen + I;
            }
          }
        }
        if (lane == 0) sm.jb = jb;
      }
      __syncthreads();
      const int jb = sm.jb;
      // add the block's tokens from its last boundary on
      if (jb >= 0) {
#pragma unroll
        for (int j = 0; j < EPT; j++) S[j] = 0.0;
      }
#pragma unroll 1
      for (int i = jb < 0 ? 0 : jb; i < nb; i++) {
        const double vi = sm.v[r0 + i][a];
#pragma unroll
        for (int j = 0; j < EPT; j += 2) {
          const double2 w = *reinterpret_cast<const double2 *>(&sm.u[r0 + i][c0 + j]);
          S[j] = fma(vi, w.x, S[j]);
          S[j + 1] = fma(vi, w.y, S[j + 1]);
        }
      }
    }
  }
  if (tid == 0 && rank == 0) {
    seg[sg] = iopen;
    aux[0] = sS;
    aux[1] = iopen;
    aux[2] = has_open ? 1.0 : 0.0;
  }
#pragma unroll
  for (int j = 0; j < EPT; j++) carry[(size_t)j * NT + tid] = S[j];
}

template <int D>
cudaError_t launch_info_d(const Dims &dm, const Plan &pl, const CallArgs &ca, cudaStream_t s) {
  const size_t sb = sizeof(InfoSmem<D>);
  cudaError_t e = cudaFuncSetAttribute(k_info_score<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sb);
  if (e != cudaSuccess) return e;
  k_info_score<D><<<2 * dm.heads, 2 * D, sb, s>>>(dm, pl, ca);  // a cluster of two CTAs per head
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_info_score(const Dims &dm, const Plan &pl, const CallArgs &ca, cudaStream_t s) {
  if (!ca.info_S || !ca.info_aux || !pl.seg_info) return cudaErrorInvalidValue;
  switch (dm.D) {
    case 32: return launch_info_d<32>(dm, pl, ca, s);
    case 64: return launch_info_d<64>(dm, pl, ca, s);
    case 128: return launch_info_d<128>(dm, pl, ca, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace dla
