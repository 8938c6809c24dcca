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
constexpr int TOKC = 16;     // tokens per ADD chunk
constexpr int OPBUF = 1024;  // ops staged in shared memory at a time

__device__ __forceinline__ void cp_async16(void *dst, const void *src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                   static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
               "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_group 0;" ::: "memory");
}


// Latency hiding: the op list is known before the replay, so the k / v rows
// of the next ADD chunk (in op order, across ops) are always in flight into a
// double-buffered raw staging area, and the next ADDP piece is preloaded into
// registers.  Both are read-only inputs of this kernel, so reading them early
// is safe.  The arithmetic per element is the same as a plain replay.
template <int D, int R, bool BF16VER>
__global__ void __launch_bounds__(THREADS) k_materialize(Dims dm, Plan pl, CallArgs ca) {
  constexpr int PER = R * D / THREADS;  // consecutive elements of one row per thread
  static_assert(R * D % THREADS == 0 && D % PER == 0 && PER % 4 == 0, "row block must split evenly");
  constexpr int RAW = TOKC * (D + R) * 4;  // k rows then v rows, fp32-sized
  const int u = blockIdx.y;
  const int r0 = blockIdx.x * R;
  const int tid = threadIdx.x;
  const int rr = (tid * PER) / D;  // row inside the block
  const int c0 = (tid * PER) % D;  // first column
  __shared__ __align__(16) uint8_t s_raw[2][RAW];
  __shared__ float s_phik[TOKC][D];
  __shared__ float s_v[TOKC][R];
  __shared__ int4 s_ops[OPBUF];
  const int4 *ops = pl.ops + (size_t)u * dm.opsmax;
  const int nops = pl.nops[u];
  float *Sbase = ca.cache.S + (size_t)u * dm.C * D * D;
  const size_t my = (size_t)(r0 + rr) * D + c0;  // element offset inside a slot
  const bool bf_in = ca.in_dtype == DLA_BF16;
  const int esz = bf_in ? 2 : 4;
  const uint8_t *kin = static_cast<const uint8_t *>(ca.k);
  const uint8_t *vin = static_cast<const uint8_t *>(ca.v);
  const size_t head_row0 = (size_t)u * dm.T + ca.w0;
  const float *pieces = pl.pieces ? pl.pieces + (size_t)u * dm.pmax * D * D + my : nullptr;
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

  int staged_end = 0;  // ops [.., staged_end) are in s_ops
  auto find_op = [&](int code, int from) -> int {
    for (int i = from; i < staged_end; i++)
      if (s_ops[i % OPBUF].x == code) return i;
    return -1;
  };
  // ---- ADD chunks: (op, chunk) in flight ----
  int inf_op = -1, inf_ch = 0, inf_buf = 0, next_buf = 0;
  auto issue_chunk = [&](int oi, int ch) {
    const int4 op = s_ops[oi % OPBUF];
    const int nt = min(TOKC, op.w - ch * TOKC);
    const size_t row0 = head_row0 + op.z + ch * TOKC;
    const int kq = D * esz / 16, vq = R * esz / 16, per_tok = kq + vq;
    uint8_t *dst = s_raw[next_buf];
    for (int e = tid; e < nt * per_tok; e += THREADS) {
      const int s = e / per_tok, w = e % per_tok;
      if (w < kq)
        cp_async16(dst + (size_t)s * D * esz + w * 16, kin + (row0 + s) * D * esz + w * 16);
      else
        cp_async16(dst + (size_t)TOKC * D * esz + (size_t)s * R * esz + (w - kq) * 16,
                   vin + ((row0 + s) * D + r0) * esz + (w - kq) * 16);
    }
    cp_async_commit();
    inf_op = oi;
    inf_ch = ch;
    inf_buf = next_buf;
    next_buf ^= 1;
  };
  // ---- ADDP pieces: the next one preloaded in registers ----
  float pfv[PER];
  int pf_op = -1;
  auto preload_piece = [&](int from) {
    pf_op = find_op(OP_ADDP, from);
    if (pf_op >= 0) {
      const float *pc = pieces + (size_t)s_ops[pf_op % OPBUF].z * D * D;
#pragma unroll
      for (int i = 0; i < PER; i += 4) {
        const float4 x = *reinterpret_cast<const float4 *>(pc + i);
        pfv[i] = x.x;
        pfv[i + 1] = x.y;
        pfv[i + 2] = x.z;
        pfv[i + 3] = x.w;
      }
    }
  };

  for (int oi = 0; oi < nops; oi++) {
    if ((oi % OPBUF) == 0) {  // stage the next ops in shared memory
      __syncthreads();
      staged_end = min(nops, oi + OPBUF);
      for (int i = tid; i < staged_end - oi; i += THREADS) s_ops[i] = ops[oi + i];
      __syncthreads();
      if (inf_op < 0) {
        const int f = find_op(OP_ADD, oi);
        if (f >= 0) issue_chunk(f, 0);
      }
      if (pf_op < 0 && pieces) preload_piece(oi);
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
      if (pf_op != oi) preload_piece(oi);
#pragma unroll
      for (int i = 0; i < PER; i++) open[i] += pfv[i];
      preload_piece(oi + 1);
    } else {  // OP_ADD: tokens [op.z, op.z + op.w) of the window into the open state
      const int nchunk = (op.w + TOKC - 1) / TOKC;
      for (int ch = 0; ch < nchunk; ch++) {
        if (inf_op != oi || inf_ch != ch) issue_chunk(oi, ch);
        const int b = inf_buf;
        cp_async_wait_all();
        __syncthreads();  // chunk visible; the previous chunk's readers are done
        inf_op = -1;
        // the following chunk in op order goes in flight now
        if (ch + 1 < nchunk) {
          issue_chunk(oi, ch + 1);
        } else {
          const int f = find_op(OP_ADD, oi + 1);
          if (f >= 0) issue_chunk(f, 0);
        }
        const int nt = min(TOKC, op.w - ch * TOKC);
        const uint8_t *rk = s_raw[b];
        const uint8_t *rv = s_raw[b] + (size_t)TOKC * D * esz;
        for (int e = tid; e < nt * D; e += THREADS) {
          const float x = bf_in ? __uint_as_float((uint32_t)reinterpret_cast<const uint16_t *>(rk)[e] << 16)
                                : reinterpret_cast<const float *>(rk)[e];
          // fast exponential: the result feeds fp32 accumulation, and its
          // error (a few ulp) is far below the state's rounding
          s_phik[e / D][e % D] = x > 0.f ? x + 1.f : __expf(x);
        }
        for (int e = tid; e < nt * R; e += THREADS)
          s_v[e / R][e % R] = bf_in ? __uint_as_float((uint32_t)reinterpret_cast<const uint16_t *>(rv)[e] << 16)
                                    : reinterpret_cast<const float *>(rv)[e];
        __syncthreads();
        for (int s = 0; s < nt; s++) {
          const float vv = s_v[s][rr];
#pragma unroll
          for (int i = 0; i < PER; i++) open[i] = fmaf(vv, s_phik[s][c0 + i], open[i]);
        }
      }
    }
  }
  cp_async_wait_all();
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
