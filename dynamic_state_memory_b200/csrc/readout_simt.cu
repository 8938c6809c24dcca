// readout_simt.cu -- fp32 SIMT readout of one tile of M tokens.
//
// o_t = sum_i lambda_{t,i} S_i phi(q_t),
// lambda_{t,i} = softmax_i(phi(q_t) . mu_i / sqrt(d_k))
// (Dynamic Linear Attention | Chlience Paper Archive, section 5.3, with the
// softmax weights fixed for this implementation).
//
// A tile starts with m0 "atoms": the states present just before its first
// token (frozen versions; the last one is the open state's partial sum).  The
// tile's tokens form pieces between in-tile boundaries.  At token t every
// state is a contiguous run of atoms and pieces (pieces only up to t's own,
// counted up to t), so with x_beta(t) = phi(q_t) . (sum of phi(k) of atom or
// piece beta up to t) and n_beta(t) its token count,
//   a_i(t) = sum_{beta in i} x_beta / (sum_{beta in i} n_beta * sqrt(d_k)),
//   o_t = sum_{atoms alpha} W_alpha(t) S_alpha phi(q_t)
//       + sum_{s <= t in tile} W_{piece(s)}(t) (phi(k_s) . phi(q_t)) v_s,
// where W_beta(t) = lambda of the state containing beta at t.  The partition
// of atoms/pieces into states only changes at in-tile boundaries ("epochs")
// and is replayed from the engine's events.
#include "dla_internal.cuh"

namespace dla {
namespace {

constexpr int THREADS = 256;
constexpr int M = 64;  // tokens per tile

struct Smem {
  float *Pq, *Kp, *Vs, *A, *X;
  uint32_t *bits;
  int *pst, *pen, *pidx;
  int BW;
};

template <int D>
__global__ void __launch_bounds__(THREADS) k_readout(Dims dm, Plan pl, CallArgs ca) {
  extern __shared__ __align__(16) float smem[];
  const int u = blockIdx.y, c = blockIdx.x;
  const int T0 = c * M;
  const int Tw = tw_of(ca, u);
  if (T0 >= Tw) return;
  const int len = min(M, Tw - T0);
  const int tid = threadIdx.x;
  const int C = dm.C;
  const int BW = (C + M + 31) / 32;
  Smem sm;
  sm.Pq = smem;
  sm.Kp = sm.Pq + M * D;
  sm.Vs = sm.Kp + M * D;
  sm.A = sm.Vs + M * D;
  sm.X = sm.A + M * (M + 1);
  sm.bits = reinterpret_cast<uint32_t *>(sm.X + (C + M) * M);
  sm.pst = reinterpret_cast<int *>(sm.bits + (M + 1) * BW);
  sm.pen = sm.pst + (M + 1);
  sm.pidx = sm.pen + (M + 1);  // [M] piece of each token
  __shared__ int s_np;

  const int m0 = pl.tile_m0[(size_t)u * dm.tiles + c];
  const int nev = pl.tile_nev[(size_t)u * dm.tiles + c];
  const int32_t *evo = pl.tile_ev_off + ((size_t)u * dm.tiles + c) * dm.M;
  const int32_t *evm = pl.tile_ev_mrg + ((size_t)u * dm.tiles + c) * dm.M;
  const int32_t *atoms = pl.tile_atoms + ((size_t)u * dm.tiles + c) * dm.amax;
  const float *ver_z = pl.ver_z + (size_t)u * dm.vmax * D;
  const float *ver_n = pl.ver_n + (size_t)u * dm.vmax;
  const float *ver_S = static_cast<const float *>(pl.ver_S) + (size_t)u * dm.vmax * D * D;

  // ---- 1. load phi(q), phi(k), v; pieces and epoch partitions ------------
  const size_t row0 = (size_t)u * dm.T + ca.w0 + T0;
  for (int e = tid; e < M * D; e += THREADS) {
    const int t = e / D, cc = e % D;
    float q = 0.f, k = 0.f, v = 0.f;
    if (t < len) {
      q = phi32(load_in(ca.q, ca.in_dtype, (row0 + t) * D + cc));
      k = phi32(load_in(ca.k, ca.in_dtype, (row0 + t) * D + cc));
      v = load_in(ca.v, ca.in_dtype, (row0 + t) * D + cc);
    }
    sm.Pq[e] = q;
    sm.Kp[e] = k;
    sm.Vs[e] = v;
  }
  if (tid == 0) {
    const bool cont = !(nev > 0 && evo[0] == 0);
    int np = 0;
    if (cont) {
      sm.pst[0] = 0;
      np = 1;
    }
    for (int i = 0; i < nev; i++) sm.pst[np++] = evo[i];
    for (int p = 0; p < np; p++) sm.pen[p] = p + 1 < np ? sm.pst[p + 1] : len;
    s_np = np;
    // epoch partitions: bit beta set = beta is the last atom/piece of a state
    uint32_t cur[16];
    for (int w = 0; w < BW; w++) cur[w] = 0;
    for (int a = 0; a < m0; a++) cur[a >> 5] |= 1u << (a & 31);
    for (int p = 0; p < np; p++) {
      const int beta = m0 + p;
      if (p == 0 && cont) {
        // the open state (last atom) continues into piece 0
        if (m0 > 0) cur[(m0 - 1) >> 5] &= ~(1u << ((m0 - 1) & 31));
      } else {
        const int code = evm[p - (cont ? 1 : 0)];
        int nm = 0, pos = -1;
        if (code >= 0) {
          nm = 1;
          pos = code;
        } else if (code <= -2) {
          nm = -code - 1;
        }
        for (int r = 0; r < nm; r++) {
          // states = set bits in order; merging pair (i, i+1) clears state i's
          // last bit.  pos < 0: the two newest states.
          int total = 0;
          for (int w = 0; w < BW; w++) total += __popc(cur[w]);
          const int i = pos >= 0 ? pos : total - 2;
          int seen = 0;
          for (int w = 0; w < BW; w++) {
            const int pc = __popc(cur[w]);
            if (i < seen + pc) {
              uint32_t x = cur[w];
              for (int k2 = 0; k2 < i - seen; k2++) x &= x - 1;
              cur[w] &= ~(x & (~x + 1));
              break;
            }
            seen += pc;
          }
        }
      }
      cur[beta >> 5] |= 1u << (beta & 31);
      for (int w = 0; w < BW; w++) sm.bits[p * BW + w] = cur[w];
    }
    for (int p = 0; p < np; p++)
      for (int t = sm.pst[p]; t < sm.pen[p]; t++) sm.pidx[t] = p;
  }
  __syncthreads();
  const int np = s_np;

  // ---- 2. A = phi(Q) phi(K)^T --------------------------------------------
  {
    const int ty = tid / 16, tx = tid % 16;  // rows ty*4.., cols tx + 16 j
    float acc[4][4] = {};
    for (int kk = 0; kk < D; kk++) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; i++) a[i] = sm.Pq[(ty * 4 + i) * D + kk];
#pragma unroll
      for (int j = 0; j < 4; j++) b[j] = sm.Kp[(tx + 16 * j) * D + kk];
#pragma unroll
      for (int i = 0; i < 4; i++)
#pragma unroll
        for (int j = 0; j < 4; j++) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
#pragma unroll
    for (int i = 0; i < 4; i++)
#pragma unroll
      for (int j = 0; j < 4; j++) sm.A[(ty * 4 + i) * (M + 1) + tx + 16 * j] = acc[i][j];
  }
  __syncthreads();
  // ---- 3. atom logits X[alpha][t] = phi(q_t) . mu_alpha --------------------
  for (int a0 = 0; a0 < m0; a0 += M) {
    const int na = min(M, m0 - a0);
    for (int e = tid; e < na * D; e += THREADS)
      sm.Kp[e] = ver_z[(size_t)atoms[a0 + e / D] * D + e % D] / ver_n[atoms[a0 + e / D]];
    __syncthreads();
    for (int e = tid; e < na * M; e += THREADS) {
      const int al = e / M, t = e % M;
      float s = 0.f;
      for (int kk = 0; kk < D; kk++) s = fmaf(sm.Pq[t * D + kk], sm.Kp[al * D + kk], s);
      sm.X[(a0 + al) * M + t] = s;
    }
    __syncthreads();
  }
  // ---- 4. per-row softmax over the states of the row's epoch -------------
  if (tid < len) {
    const int t = tid;
    const int ep = sm.pidx[t];
    const float inv_sqrt_d = 1.0f / sqrtf((float)D);
    const uint32_t *bits = sm.bits + ep * BW;
    float sacc = 0.f, nacc = 0.f, mx = -INFINITY, l = 0.f;
    for (int beta = 0; beta <= m0 + ep; beta++) {
      float x, nn;
      if (beta < m0) {
        nn = ver_n[atoms[beta]];
        x = nn * sm.X[beta * M + t];
      } else {
        const int p = beta - m0;
        const int s1 = p == ep ? t + 1 : sm.pen[p];
        x = 0.f;
        for (int s = sm.pst[p]; s < s1; s++) x += sm.A[t * (M + 1) + s];
        nn = (float)(s1 - sm.pst[p]);
      }
      sacc += x;
      nacc += nn;
      if (bits[beta >> 5] >> (beta & 31) & 1u) {
        const float a = sacc / nacc * inv_sqrt_d;
        sm.X[beta * M + t] = a;
        const float nmx = fmaxf(mx, a);
        l = l * __expf(mx - nmx) + __expf(a - nmx);
        mx = nmx;
        sacc = 0.f;
        nacc = 0.f;
      }
    }
    float cur = 0.f;
    for (int beta = m0 + ep; beta >= 0; beta--) {
      if (bits[beta >> 5] >> (beta & 31) & 1u) cur = expf(sm.X[beta * M + t] - mx) / l;
      sm.X[beta * M + t] = cur;
    }
    for (int beta = m0 + ep + 1; beta < m0 + np; beta++) sm.X[beta * M + t] = 0.f;
    // intra-tile weights: A[t][s] *= W_{piece(s)}(t) for s <= t, 0 beyond
    for (int s = 0; s < M; s++) {
      const float w = (s <= t) ? sm.X[(m0 + sm.pidx[s]) * M + t] : 0.f;
      sm.A[t * (M + 1) + s] *= w;
    }
  } else if (tid < M) {
    for (int s = 0; s < M; s++) sm.A[tid * (M + 1) + s] = 0.f;
    for (int beta = 0; beta < m0 + np; beta++) sm.X[beta * M + tid] = 0.f;
  }
  __syncthreads();
  // ---- 5. o = sum_alpha W_alpha S_alpha phi(q) + (W o A) V -----------------
  const int ty = tid / 16, tx = tid % 16;  // rows ty*4 + i, cols tx + 16 j
  constexpr int NC = D / 16;
  float o[4][NC];
#pragma unroll
  for (int i = 0; i < 4; i++)
#pragma unroll
    for (int j = 0; j < NC; j++) o[i][j] = 0.f;
  constexpr int KC = 32;  // k chunk of S staged in smem (D rows x KC)
  float *Ss = sm.Kp;      // D * KC floats <= M * D
  for (int al = 0; al < m0; al++) {
    const float *S = ver_S + (size_t)atoms[al] * D * D;
    float p[4][NC];
#pragma unroll
    for (int i = 0; i < 4; i++)
#pragma unroll
      for (int j = 0; j < NC; j++) p[i][j] = 0.f;
    for (int k0 = 0; k0 < D; k0 += KC) {
      __syncthreads();
      for (int e = tid; e < D * KC; e += THREADS) {
        const int r = e / KC, kk = e % KC;
        Ss[r * (KC + 1) + kk] = S[(size_t)r * D + k0 + kk];
      }
      __syncthreads();
      for (int kk = 0; kk < KC; kk++) {
        float a[4];
#pragma unroll
        for (int i = 0; i < 4; i++) a[i] = sm.Pq[(ty * 4 + i) * D + k0 + kk];
#pragma unroll
        for (int j = 0; j < NC; j++) {
          const float b = Ss[(tx + 16 * j) * (KC + 1) + kk];
#pragma unroll
          for (int i = 0; i < 4; i++) p[i][j] = fmaf(a[i], b, p[i][j]);
        }
      }
    }
#pragma unroll
    for (int i = 0; i < 4; i++) {
      const float w = sm.X[al * M + ty * 4 + i];
#pragma unroll
      for (int j = 0; j < NC; j++) o[i][j] = fmaf(w, p[i][j], o[i][j]);
    }
  }
  for (int s = 0; s < M; s++) {
    float a[4];
#pragma unroll
    for (int i = 0; i < 4; i++) a[i] = sm.A[(ty * 4 + i) * (M + 1) + s];
#pragma unroll
    for (int j = 0; j < NC; j++) {
      const float b = sm.Vs[s * D + tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; i++) o[i][j] = fmaf(a[i], b, o[i][j]);
    }
  }
#pragma unroll
  for (int i = 0; i < 4; i++) {
    const int t = ty * 4 + i;
    if (t < len)
#pragma unroll
      for (int j = 0; j < NC; j++) store_out(ca.o, ca.in_dtype, (row0 + t) * D + tx + 16 * j, o[i][j]);
  }
}

template <int D>
size_t smem_bytes(int C) {
  const int BW = (C + M + 31) / 32;
  return sizeof(float) * (3 * M * D + M * (M + 1) + (C + M) * M) +
         sizeof(uint32_t) * (M + 1) * BW + sizeof(int) * (3 * (M + 1));
}

template <int D>
cudaError_t launch_d(const Dims &dm, const Plan &pl, const CallArgs &ca, cudaStream_t s) {
  const size_t sb = smem_bytes<D>(dm.C);
  cudaError_t e = cudaFuncSetAttribute(k_readout<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)sb);
  if (e != cudaSuccess) return e;
  dim3 g(dm.tiles, dm.heads);
  k_readout<D><<<g, THREADS, sb, s>>>(dm, pl, ca);
  return cudaGetLastError();
}

}  // namespace

int simt_tile_rows() { return M; }

// Whether a tile's atoms (up to C) fit the SIMT readout's shared memory and
// its epoch bitmask.
bool simt_fits(int D, int C) {
  if (C + M > 16 * 32) return false;
  size_t b = 0;
  switch (D) {
    case 32: b = smem_bytes<32>(C); break;
    case 64: b = smem_bytes<64>(C); break;
    case 128: b = smem_bytes<128>(C); break;
    default: return false;
  }
  return b <= 227 * 1024;
}

cudaError_t launch_readout_simt(const Dims &dm, const Plan &pl, const CallArgs &ca,
                                cudaStream_t s) {
  if (dm.M != M || dm.C + M > 16 * 32) return cudaErrorInvalidValue;
  switch (dm.D) {
    case 32: return launch_d<32>(dm, pl, ca, s);
    case 64: return launch_d<64>(dm, pl, ca, s);
    case 128: return launch_d<128>(dm, pl, ca, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace dla
