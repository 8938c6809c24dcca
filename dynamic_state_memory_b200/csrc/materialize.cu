// materialize.cu -- executes the engine's op list on the fp32 slot states.
//
// Each CTA owns R rows (of d_v) of every slot of one head and replays the
// head's ops in order, so no two CTAs touch the same element and no
// inter-CTA synchronisation is needed:
//   ZERO(slot)            S_slot = 0                 (a new open state)
//   ADD(slot, t, cnt)     S_slot += v_s phi(k_s)^T   for cnt tokens from t
//                         (Chlience section 5.1: the per-token state joins the
//                          current state)
//   MERGE(dst, src)       S_dst += S_src             (Chlience section 5.2)
//   SHADOW(slot, ver)     version ver = S_slot, frozen for the readout
//                         (fp32 copy, or bf16 in the tensor-core tile layout)
#include "dla_internal.cuh"

namespace dla {
namespace {

constexpr int THREADS = 256;
constexpr int TOK = 32;  // tokens staged per ADD step

template <int D, int R, bool BF16VER>
__global__ void __launch_bounds__(THREADS) k_materialize(Dims dm, Plan pl, CallArgs ca) {
  constexpr int PER = R * D / THREADS;  // elements per thread
  static_assert(R * D % THREADS == 0, "row block must split evenly");
  const int u = blockIdx.y;
  const int r0 = blockIdx.x * R;
  const int tid = threadIdx.x;
  __shared__ float s_phik[TOK][D];
  __shared__ float s_v[TOK][R];
  const int4 *ops = pl.ops + (size_t)u * dm.opsmax;
  const int nops = pl.nops[u];
  float *Sbase = ca.cache.S + (size_t)u * dm.C * D * D;
  for (int oi = 0; oi < nops; oi++) {
    const int4 op = ops[oi];
    float *Sa = Sbase + ((size_t)op.y * D + r0) * D;
    if (op.x == OP_ZERO) {
#pragma unroll
      for (int i = 0; i < PER; i++) Sa[tid + THREADS * i] = 0.0f;
    } else if (op.x == OP_MERGE) {
      const float *Sb = Sbase + ((size_t)op.z * D + r0) * D;
#pragma unroll
      for (int i = 0; i < PER; i++) Sa[tid + THREADS * i] += Sb[tid + THREADS * i];
    } else if (op.x == OP_SHADOW) {
      if (BF16VER) {
        // handled by the tensor-core path's own materializer
      } else {
        float *Vd = static_cast<float *>(pl.ver_S) + (((size_t)u * dm.vmax + op.z) * D + r0) * D;
#pragma unroll
        for (int i = 0; i < PER; i++) Vd[tid + THREADS * i] = Sa[tid + THREADS * i];
      }
    } else {  // OP_ADD
      float acc[PER];
#pragma unroll
      for (int i = 0; i < PER; i++) acc[i] = Sa[tid + THREADS * i];
      const size_t row0 = (size_t)u * dm.T + ca.w0 + op.z;
      for (int s0 = 0; s0 < op.w; s0 += TOK) {
        const int nt = min(TOK, op.w - s0);
        __syncthreads();
        for (int e = tid; e < nt * D; e += THREADS) {
          const int s = e / D, c = e % D;
          s_phik[s][c] = phi32(load_in(ca.k, ca.in_dtype, (row0 + s0 + s) * D + c));
        }
        for (int e = tid; e < nt * R; e += THREADS) {
          const int s = e / R, rr = e % R;
          s_v[s][rr] = load_in(ca.v, ca.in_dtype, (row0 + s0 + s) * D + r0 + rr);
        }
        __syncthreads();
        for (int s = 0; s < nt; s++) {
#pragma unroll
          for (int i = 0; i < PER; i++) {
            const int e = tid + THREADS * i;
            acc[i] = fmaf(s_v[s][e / D], s_phik[s][e % D], acc[i]);
          }
        }
      }
#pragma unroll
      for (int i = 0; i < PER; i++) Sa[tid + THREADS * i] = acc[i];
    }
  }
}

template <int D>
cudaError_t launch_d(const Dims &dm, const Plan &pl, const CallArgs &ca, cudaStream_t s) {
  constexpr int R = (D * D < 2048) ? D : 2048 / D;
  dim3 g(D / R, dm.heads);
  k_materialize<D, R, false><<<g, THREADS, 0, s>>>(dm, pl, ca);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_materialize(const Dims &dm, const Plan &pl, const CallArgs &ca,
                               cudaStream_t s) {
  switch (dm.D) {
    case 32: return launch_d<32>(dm, pl, ca, s);
    case 64: return launch_d<64>(dm, pl, ca, s);
    case 128: return launch_d<128>(dm, pl, ca, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace dla
