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
#include "tc_ptx.cuh"

namespace dla {
namespace {

constexpr int THREADS = 256;
constexpr int TOK = 32;  // tokens staged per ADD step

template <int D, int R, bool BF16VER>
__global__ void __launch_bounds__(THREADS) k_materialize(Dims dm, Plan pl, CallArgs ca) {
  constexpr int PER = R * D / THREADS;  // consecutive elements of one row per thread
  static_assert(R * D % THREADS == 0 && D % PER == 0, "row block must split evenly");
  const int u = blockIdx.y;
  const int r0 = blockIdx.x * R;
  const int tid = threadIdx.x;
  const int rr = (tid * PER) / D;       // row inside the block
  const int c0 = (tid * PER) % D;       // first column
  __shared__ float s_phik[TOK][D];
  __shared__ float s_v[TOK][R];
  const int4 *ops = pl.ops + (size_t)u * dm.opsmax;
  const int nops = pl.nops[u];
  float *Sbase = ca.cache.S + (size_t)u * dm.C * D * D;
  const size_t my = (size_t)(r0 + rr) * D + c0;  // element offset inside a slot
  for (int oi = 0; oi < nops; oi++) {
    const int4 op = ops[oi];
    float *Sa = Sbase + (size_t)op.y * D * D + my;
    if (op.x == OP_ZERO) {
#pragma unroll
      for (int i = 0; i < PER; i += 4) *reinterpret_cast<float4 *>(Sa + i) = make_float4(0.f, 0.f, 0.f, 0.f);
    } else if (op.x == OP_MERGE) {
      const float *Sb = Sbase + (size_t)op.z * D * D + my;
#pragma unroll
      for (int i = 0; i < PER; i += 4) {
        float4 a = *reinterpret_cast<const float4 *>(Sa + i);
        const float4 b = *reinterpret_cast<const float4 *>(Sb + i);
        a.x += b.x;
        a.y += b.y;
        a.z += b.z;
        a.w += b.w;
        *reinterpret_cast<float4 *>(Sa + i) = a;
      }
    } else if (op.x == OP_SHADOW) {
      if constexpr (BF16VER) {
        // bf16 version in the UMMA K-major 128-byte-swizzle layout (rows d_v)
        uint8_t *Vd = static_cast<uint8_t *>(pl.ver_S) + ((size_t)u * dm.vmax + op.z) * D * D * 2;
        uint32_t w[PER / 2];
#pragma unroll
        for (int i = 0; i < PER; i += 2) w[i / 2] = tc::pack_bf16(Sa[i], Sa[i + 1]);
        static_assert(!BF16VER || PER == 8, "one 16-byte chunk per thread");
        *reinterpret_cast<uint4 *>(Vd + tc::sw128_offset(r0 + rr, c0, D)) = make_uint4(w[0], w[1], w[2], w[3]);
      } else {
        float *Vd = static_cast<float *>(pl.ver_S) + ((size_t)u * dm.vmax + op.z) * D * D + my;
#pragma unroll
        for (int i = 0; i < PER; i += 4) *reinterpret_cast<float4 *>(Vd + i) = *reinterpret_cast<const float4 *>(Sa + i);
      }
    } else {  // OP_ADD
      float acc[PER];
#pragma unroll
      for (int i = 0; i < PER; i++) acc[i] = Sa[i];
      const size_t row0 = (size_t)u * dm.T + ca.w0 + op.z;
      for (int s0 = 0; s0 < op.w; s0 += TOK) {
        const int nt = min(TOK, op.w - s0);
        __syncthreads();
        for (int e = tid; e < nt * D; e += THREADS) {
          const int s = e / D, c = e % D;
          s_phik[s][c] = phi32(load_in(ca.k, ca.in_dtype, (row0 + s0 + s) * D + c));
        }
        for (int e = tid; e < nt * R; e += THREADS) {
          const int s = e / R, r = e % R;
          s_v[s][r] = load_in(ca.v, ca.in_dtype, (row0 + s0 + s) * D + r0 + r);
        }
        __syncthreads();
        for (int s = 0; s < nt; s++) {
          const float vv = s_v[s][rr];
#pragma unroll
          for (int i = 0; i < PER; i++) acc[i] = fmaf(vv, s_phik[s][c0 + i], acc[i]);
        }
      }
#pragma unroll
      for (int i = 0; i < PER; i++) Sa[i] = acc[i];
    }
  }
}

template <int D>
cudaError_t launch_d(const Dims &dm, const Plan &pl, const CallArgs &ca, cudaStream_t s,
                     bool bf16_versions) {
  constexpr int R = (D * D < 2048) ? D : 2048 / D;
  dim3 g(D / R, dm.heads);
  if constexpr (D == 128) {
    if (bf16_versions) {
      k_materialize<D, R, true><<<g, THREADS, 0, s>>>(dm, pl, ca);
      return cudaGetLastError();
    }
  }
  if (bf16_versions) return cudaErrorInvalidValue;
  k_materialize<D, R, false><<<g, THREADS, 0, s>>>(dm, pl, ca);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_materialize(const Dims &dm, const Plan &pl, const CallArgs &ca,
                               cudaStream_t s, bool bf16_versions) {
  switch (dm.D) {
    case 32: return launch_d<32>(dm, pl, ca, s, bf16_versions);
    case 64: return launch_d<64>(dm, pl, ca, s, bf16_versions);
    case 128: return launch_d<128>(dm, pl, ca, s, bf16_versions);
  }
  return cudaErrorInvalidValue;
}

}  // namespace dla
