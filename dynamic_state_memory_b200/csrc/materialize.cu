// materialize.cu -- executes the engine's op list on the fp32 slot states.
//
// Each CTA owns R rows (of d_v) of every slot of one head and replays the
// head's ops in order, so no two CTAs touch the same element and no
// inter-CTA synchronisation is needed.  The open state lives in registers:
//   ZERO(slot) / LOAD(slot)   the open state starts at 0 / from its slot
//   ADD(slot, t, cnt)         open += v_s phi(k_s)^T for cnt tokens from t
//                             (Chlience section 5.1: the per-token state joins
//                             the current state)
//   ADDP(slot, piece)         open += the tensor-core builder's piece
//   STORE(slot, -, ver + 1)   S_slot = open (the state is sealed)
//   MERGE(dst, src, ver + 1)  S_dst += S_src             (Chlience section 5.2)
//   MERGEO(dst, -, ver + 1)   S_dst += open (the just-sealed state merges left)
//   SHADOW(slot, ver)         version ver = S_slot (or the open registers)
// A non-zero .w of STORE / MERGE / MERGEO also freezes the result as version
// .w - 1 from registers (fp32 copy, or bf16 in the tensor-core tile layout).
#include "dla_internal.cuh"
#include "tc_ptx.cuh"

namespace dla {
namespace {

constexpr int THREADS = 256;
constexpr int TOK = 32;  // tokens staged per ADD step

template <int D, int R, bool BF16VER>
__global__ void __launch_bounds__(THREADS) k_materialize(Dims dm, Plan pl, CallArgs ca) {
  constexpr int PER = R * D / THREADS;  // consecutive elements of one row per thread
  static_assert(R * D % THREADS == 0 && D % PER == 0 && PER % 4 == 0, "row block must split evenly");
  constexpr int KPT = TOK * D / THREADS;  // k values staged per thread per chunk
  constexpr int VPT = (TOK * R + THREADS - 1) / THREADS;
  const int u = blockIdx.y;
  const int r0 = blockIdx.x * R;
  const int tid = threadIdx.x;
  const int rr = (tid * PER) / D;  // row inside the block
  const int c0 = (tid * PER) % D;  // first column
  __shared__ float s_phik[2][TOK][D];
  __shared__ float s_v[2][TOK][R];
  constexpr int OPBUF = 512;
  __shared__ int4 s_ops[OPBUF];
  const int4 *ops = pl.ops + (size_t)u * dm.opsmax;
  const int nops = pl.nops[u];
  float *Sbase = ca.cache.S + (size_t)u * dm.C * D * D;
  const size_t my = (size_t)(r0 + rr) * D + c0;  // element offset inside a slot
  float open[PER];
  int open_slot = -1;
#pragma unroll
  for (int i = 0; i < PER; i++) open[i] = 0.f;
  auto shadow = [&](int v, const float *src) {
    if constexpr (BF16VER) {
      uint8_t *Vd = static_cast<uint8_t *>(pl.ver_S) + ((size_t)u * dm.vmax + v) * D * D * 2;
#pragma unroll
      for (int i = 0; i < PER; i += 8)
        *reinterpret_cast<uint4 *>(Vd + tc::sw128_offset(r0 + rr, c0 + i, D)) =
            make_uint4(tc::pack_bf16(src[i], src[i + 1]), tc::pack_bf16(src[i + 2], src[i + 3]),
                       tc::pack_bf16(src[i + 4], src[i + 5]), tc::pack_bf16(src[i + 6], src[i + 7]));
    } else {
      float *Vd = static_cast<float *>(pl.ver_S) + ((size_t)u * dm.vmax + v) * D * D + my;
#pragma unroll
      for (int i = 0; i < PER; i += 4)
        *reinterpret_cast<float4 *>(Vd + i) = make_float4(src[i], src[i + 1], src[i + 2], src[i + 3]);
    }
  };
  for (int oi = 0; oi < nops; oi++) {
    if ((oi % OPBUF) == 0) {  // stage the next ops in shared memory
      __syncthreads();
      for (int i = tid; i < OPBUF && oi + i < nops; i += THREADS) s_ops[i] = ops[oi + i];
      __syncthreads();
    }
    const int4 op = s_ops[oi % OPBUF];
    float *Sa = Sbase + (size_t)op.y * D * D + my;
    if (op.x == OP_ZERO) {
      open_slot = op.y;
#pragma unroll
      for (int i = 0; i < PER; i++) open[i] = 0.f;
    } else if (op.x == OP_LOAD) {
      open_slot = op.y;
#pragma unroll
      for (int i = 0; i < PER; i += 4) {
        const float4 x = *reinterpret_cast<const float4 *>(Sa + i);
        open[i] = x.x;
        open[i + 1] = x.y;
        open[i + 2] = x.z;
        open[i + 3] = x.w;
      }
    } else if (op.x == OP_STORE) {
#pragma unroll
      for (int i = 0; i < PER; i += 4)
        *reinterpret_cast<float4 *>(Sa + i) = make_float4(open[i], open[i + 1], open[i + 2], open[i + 3]);
      if (op.w > 0) shadow(op.w - 1, open);
      open_slot = -1;
    } else if (op.x == OP_MERGE || op.x == OP_MERGEO) {
      const float *Sb = Sbase + (size_t)op.z * D * D + my;
      float sum[PER];
#pragma unroll
      for (int i = 0; i < PER; i += 4) {
        const float4 a = *reinterpret_cast<const float4 *>(Sa + i);
        float4 b;
        if (op.x == OP_MERGE) b = *reinterpret_cast<const float4 *>(Sb + i);
        else b = make_float4(open[i], open[i + 1], open[i + 2], open[i + 3]);
        sum[i] = a.x + b.x;
        sum[i + 1] = a.y + b.y;
        sum[i + 2] = a.z + b.z;
        sum[i + 3] = a.w + b.w;
        *reinterpret_cast<float4 *>(Sa + i) = make_float4(sum[i], sum[i + 1], sum[i + 2], sum[i + 3]);
      }
      if (op.w > 0) shadow(op.w - 1, sum);
      if (op.x == OP_MERGEO) open_slot = -1;
    } else if (op.x == OP_SHADOW) {
      if (op.y == open_slot) {
        shadow(op.z, open);
      } else {
        float tmp[PER];
#pragma unroll
        for (int i = 0; i < PER; i += 4) {
          const float4 x = *reinterpret_cast<const float4 *>(Sa + i);
          tmp[i] = x.x;
          tmp[i + 1] = x.y;
          tmp[i + 2] = x.z;
          tmp[i + 3] = x.w;
        }
        shadow(op.z, tmp);
      }
    } else if (op.x == OP_ADDP) {
      const float *pc = pl.pieces + ((size_t)u * dm.pmax + op.z) * D * D + my;
#pragma unroll
      for (int i = 0; i < PER; i += 4) {
        const float4 x = *reinterpret_cast<const float4 *>(pc + i);
        open[i] += x.x;
        open[i + 1] += x.y;
        open[i + 2] += x.z;
        open[i + 3] += x.w;
      }
    } else {  // OP_ADD: tokens [op.z, op.z + op.w) of the window into the open state
      const size_t row0 = (size_t)u * dm.T + ca.w0 + op.z;
      const int nchunk = (op.w + TOK - 1) / TOK;
      float kr[KPT], vr[VPT];
      auto fetch = [&](int ch) {
        const int nt = min(TOK, op.w - ch * TOK);
#pragma unroll
        for (int i = 0; i < KPT; i++) {
          const int e = tid + THREADS * i, s = e / D, c = e % D;
          kr[i] = s < nt ? load_in(ca.k, ca.in_dtype, (row0 + ch * TOK + s) * D + c) : 0.f;
        }
#pragma unroll
        for (int i = 0; i < VPT; i++) {
          const int e = tid + THREADS * i, s = e / R, r = e % R;
          vr[i] = (e < TOK * R && s < nt) ? load_in(ca.v, ca.in_dtype, (row0 + ch * TOK + s) * D + r0 + r) : 0.f;
        }
      };
      fetch(0);
      for (int ch = 0; ch < nchunk; ch++) {
        const int buf = ch & 1;
#pragma unroll
        for (int i = 0; i < KPT; i++) {
          const int e = tid + THREADS * i;
          s_phik[buf][e / D][e % D] = phi32(kr[i]);
        }
#pragma unroll
        for (int i = 0; i < VPT; i++) {
          const int e = tid + THREADS * i;
          if (e < TOK * R) s_v[buf][e / R][e % R] = vr[i];
        }
        __syncthreads();
        if (ch + 1 < nchunk) fetch(ch + 1);
        const int nt = min(TOK, op.w - ch * TOK);
        for (int s = 0; s < nt; s++) {
          const float vv = s_v[buf][s][rr];
#pragma unroll
          for (int i = 0; i < PER; i++) open[i] = fmaf(vv, s_phik[buf][s][c0 + i], open[i]);
        }
      }
      __syncthreads();
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
