// decode.cu -- one DLA decode step for every stream of a cache.
//
// k_decode_decide (one warp per stream): the token's score against the cached
//   previous key (fp64, index order, bit-identical to the CPU oracle), the
//   boundary rule, sealing, the capacity merge by least Ward loss over the
//   cached pair losses, the fp64 summary updates (z, n, ts, order), and the
//   softmax weights lambda_i = softmax_i(phi(q) . mu_i / sqrt(d)) of every
//   live state after the update.  It leaves, per stream, lambda per slot and
//   one instruction for the streaming kernel (which slot takes v phi(k)^T,
//   whether that slot is new, and the merged pair).
//   (ai-feeds.com "Dynamic Linear Attention" summary, 方法; Dynamic Linear
//   Attention | Chlience Paper Archive, sections 5.1-5.3.)
// k_decode_stream: streams each live fp32 state once with 128-bit coalesced
//   loads, applies the merge / open-state update in registers, writes back the
//   changed slots and accumulates o = sum_i lambda_i S_i phi(q).  Each CTA owns
//   32 rows of d_v of one stream, so o needs no cross-CTA reduction.
#include <cuda.h>

#include <mutex>

#include "dla_internal.cuh"

namespace dla {
namespace {

constexpr unsigned FULL = 0xffffffffu;

struct DecodeWs {
  float *lam;     // [U][C] weight of each slot (0 = not live)
  int4 *instr;    // [U] {open slot, open is new, merge dst (-1 none), merge src}
};

DecodeWs carve_ws(void *ws, int U, int C) {
  DecodeWs w;
  char *p = static_cast<char *>(ws);
  w.lam = reinterpret_cast<float *>(p);
  size_t off = ((size_t)U * C * sizeof(float) + 255) / 256 * 256;
  w.instr = reinterpret_cast<int4 *>(p + off);
  return w;
}

__device__ double ward64(const double *za, const double *zb, double na, double nb, int D,
                         int lane) {
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

__global__ void __launch_bounds__(128) k_decode_decide(dla_cache cc, float tau, int32_t dt,
                                                       const void *q, const void *k,
                                                       DecodeWs w, uint8_t *boundary,
                                                       int32_t *merge_i, int32_t *dev_status,
                                                       const uint8_t *active) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int u = blockIdx.x * 4 + warp;
  const int U = cc.N * cc.H;
  if (u >= U) return;
  if (active && !active[u / cc.H]) {
    // a sequence that takes no token this step: its cache is left alone and
    // the streaming kernel skips it (open slot -1)
    if (lane == 0) w.instr[u] = make_int4(-1, 0, -1, -1);
    return;
  }
  const int C = cc.C, D = cc.d_k;
  int32_t *order = cc.order + (size_t)u * C;
  int64_t *n = cc.n + (size_t)u * C;
  int64_t *ts = cc.ts + (size_t)u * C;
  double *z = cc.z + (size_t)u * C * D;
  double *loss = cc.pair_loss + (size_t)u * C;
  float *prev_k = cc.prev_k + (size_t)u * D;
  const int64_t t = cc.t[u];
  int m = cc.m[u];
  const size_t row = (size_t)u * D;
  // a cache of the information or unbounded policy is not continued here
  if (lane == 0 && loss[C - 1] < 0.0) set_status(dev_status, DLA_ERR_UNSUPPORTED);

  // score in index order on lane 0 (same operation sequence as the oracle)
  double r = 0.0;
  if (lane == 0 && t > 0) {
    double dot = 0.0, na = 0.0, nb = 0.0;
    for (int c = 0; c < D; c++)
      dot = __dadd_rn(dot, __dmul_rn((double)load_in(k, dt, row + c), (double)prev_k[c]));
    for (int c = 0; c < D; c++) {
      const double x = (double)load_in(k, dt, row + c);
      na = __dadd_rn(na, __dmul_rn(x, x));
    }
    for (int c = 0; c < D; c++) {
      const double y = (double)prev_k[c];
      nb = __dadd_rn(nb, __dmul_rn(y, y));
    }
    r = (na == 0.0 || nb == 0.0)
            ? 1.0
            : __dsub_rn(1.0, __ddiv_rn(dot, __dmul_rn(__dsqrt_rn(na), __dsqrt_rn(nb))));
  }
  r = __shfl_sync(FULL, r, 0);
  const bool join = t > 0 && r < (double)tau && cc.prev_r[u] < (double)tau;
  int open_new = 0, mdst = -1, msrc = -1, mi = -1;
  int open_slot;
  if (!join) {
    if (m > 0) {
      // seal the open state; its pair loss with the previous sealed state
      if (m >= 2) {
        const int sa = order[m - 2], sb = order[m - 1];
        const double l = ward64(z + (size_t)sa * D, z + (size_t)sb * D, (double)n[sa],
                                (double)n[sb], D, lane);
        if (lane == 0) loss[m - 2] = l;
      }
      __syncwarp();
      if (m == C) {
        double best = INFINITY;
        int bi = 0x7fffffff;
        for (int p = lane; p < C - 1; p += 32) {
          const double l = loss[p];
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
        const int a = order[is], b = order[is + 1];
        for (int c = lane; c < D; c += 32)
          z[(size_t)a * D + c] = __dadd_rn(z[(size_t)a * D + c], z[(size_t)b * D + c]);
        int32_t ov[4];
        double lv[4];
        for (int qq = 0; qq < 4; qq++) {
          const int p = lane + 32 * qq;
          ov[qq] = (p >= is + 1 && p + 1 < C) ? order[p + 1] : 0;
          lv[qq] = (p >= is + 1 && p + 1 < C - 1) ? loss[p + 1] : 0.0;
        }
        __syncwarp();
        if (lane == 0) n[a] += n[b];
        for (int qq = 0; qq < 4; qq++) {
          const int p = lane + 32 * qq;
          if (p >= is + 1 && p + 1 < C) order[p] = ov[qq];
          if (p >= is + 1 && p + 1 < C - 1) loss[p] = lv[qq];
        }
        __syncwarp();
        m -= 1;
        if (is >= 1) {
          const double l = ward64(z + (size_t)order[is - 1] * D, z + (size_t)order[is] * D,
                                  (double)n[order[is - 1]], (double)n[order[is]], D, lane);
          if (lane == 0) loss[is - 1] = l;
        }
        if (is + 1 <= m - 1) {
          const double l = ward64(z + (size_t)order[is] * D, z + (size_t)order[is + 1] * D,
                                  (double)n[order[is]], (double)n[order[is + 1]], D, lane);
          if (lane == 0) loss[is] = l;
        }
        __syncwarp();
        mdst = a;
        msrc = b;
        mi = is;
      }
    }
    // allocate the lowest free slot for the new open state
    uint32_t used[4] = {0, 0, 0, 0};
    for (int p = 0; p < m; p++) used[order[p] >> 5] |= 1u << (order[p] & 31);
    open_slot = 0;
    for (int wd = 0; wd < 4; wd++) {
      const uint32_t fr = ~used[wd];
      if (wd * 32 < C && fr) {
        const int s = wd * 32 + __ffs(fr) - 1;
        if (s < C) {
          open_slot = s;
          break;
        }
      }
    }
    if (lane == 0) {
      order[m] = open_slot;
      n[open_slot] = 0;
      ts[open_slot] = t;
    }
    for (int c = lane; c < D; c += 32) z[(size_t)open_slot * D + c] = 0.0;
    __syncwarp();
    m += 1;
    open_new = 1;
  } else {
    open_slot = order[m - 1];
  }
  // the token joins the open state's summaries (fp64, in token order)
  for (int c = lane; c < D; c += 32)
    z[(size_t)open_slot * D + c] = __dadd_rn(z[(size_t)open_slot * D + c],
                                             phi64((double)load_in(k, dt, row + c)));
  if (lane == 0) n[open_slot] += 1;
  __syncwarp();
  // lambda over the live states (lane per state), fp32 logits
  __shared__ float s_pq[4][128];
  for (int c = lane; c < D; c += 32) s_pq[warp][c] = phi32(load_in(q, dt, row + c));
  __syncwarp();
  const float isd = 1.0f / sqrtf((float)D);
  float av[4];
  for (int qq = 0; qq < 4; qq++) {
    const int p = lane + 32 * qq;
    float a = -INFINITY;
    if (p < m) {
      const int s = order[p];
      const float inv_n = 1.0f / (float)n[s];
      float acc = 0.f;
      for (int c = 0; c < D; c++) acc = fmaf(s_pq[warp][c], (float)z[(size_t)s * D + c] * inv_n, acc);
      a = acc * isd;
    }
    av[qq] = a;
  }
  float mx = fmaxf(fmaxf(av[0], av[1]), fmaxf(av[2], av[3]));
  for (int off = 16; off; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, off));
  float ev[4], den = 0.f;
  for (int qq = 0; qq < 4; qq++) {
    ev[qq] = (lane + 32 * qq < m) ? expf(av[qq] - mx) : 0.f;
    den += ev[qq];
  }
  for (int off = 16; off; off >>= 1) den += __shfl_xor_sync(FULL, den, off);
  float *lam = w.lam + (size_t)u * C;
  for (int s = lane; s < C; s += 32) lam[s] = 0.f;
  __syncwarp();
  for (int qq = 0; qq < 4; qq++) {
    const int p = lane + 32 * qq;
    if (p < m) lam[order[p]] = ev[qq] / den;
  }
  if (lane == 0) {
    w.instr[u] = make_int4(open_slot, open_new, mdst, msrc);
    cc.m[u] = m;
    cc.t[u] = t + 1;
    cc.prev_r[u] = r;
    if (boundary) boundary[u] = join ? 0 : 1;
    if (merge_i) merge_i[u] = mi;
    if (m > C) set_status(dev_status, DLA_ERR_INVARIANT);
  }
  for (int c = lane; c < D; c += 32) prev_k[c] = load_in(k, dt, row + c);
}

// Rows of d_v per stream are split over CTAs of 8 warps x 4 rows; a row of D
// floats is D/4 float4, one per active lane.
constexpr int ROWS_PER_WARP = 4;
constexpr int WARPS = 8;
constexpr int ROWS_PER_CTA = ROWS_PER_WARP * WARPS;

__device__ __forceinline__ float dot4(const float4 &a, const float *p) {
  return a.x * p[0] + a.y * p[1] + a.z * p[2] + a.w * p[3];
}

template <int D>
__global__ void __launch_bounds__(WARPS * 32) k_decode_stream(dla_cache cc, int32_t dt,
                                                              const void *q, const void *k,
                                                              const void *v, void *o,
                                                              DecodeWs w) {
  const int u = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r0 = blockIdx.x * ROWS_PER_CTA + warp * ROWS_PER_WARP;
  if (r0 >= D) return;
  const bool act = lane * 4 < D;
  const int ln = act ? lane : 0;
  const int C = cc.C;
  const size_t row = (size_t)u * D;
  const int4 ins = w.instr[u];
  if (ins.x < 0) return;  // an inactive sequence (masked step)
  const float *lam = w.lam + (size_t)u * C;
  const float4 z4 = make_float4(0.f, 0.f, 0.f, 0.f);
  float pq[4], pk[4], vr[ROWS_PER_WARP];
#pragma unroll
  for (int j = 0; j < 4; j++) {
    pq[j] = act ? phi32(load_in(q, dt, row + 4 * ln + j)) : 0.f;
    pk[j] = act ? phi32(load_in(k, dt, row + 4 * ln + j)) : 0.f;
  }
#pragma unroll
  for (int i = 0; i < ROWS_PER_WARP; i++) vr[i] = load_in(v, dt, row + r0 + i);
  float *S = cc.S + (size_t)u * C * D * D;
  auto at = [&](int slot, int i) {
    return reinterpret_cast<float4 *>(S + ((size_t)slot * D + r0 + i) * D) + ln;
  };
  float acc[ROWS_PER_WARP];
#pragma unroll
  for (int i = 0; i < ROWS_PER_WARP; i++) acc[i] = 0.f;
  const int open_slot = ins.x, open_new = ins.y, mdst = ins.z, msrc = ins.w;
  // merged pair: S_dst += S_src (read both, write dst) before the open state
  // may reuse the freed slot
  if (mdst >= 0) {
    float4 a[ROWS_PER_WARP], b[ROWS_PER_WARP];
#pragma unroll
    for (int i = 0; i < ROWS_PER_WARP; i++) {
      a[i] = act ? *at(mdst, i) : z4;
      b[i] = act ? *at(msrc, i) : z4;
    }
    const float l = lam[mdst];
#pragma unroll
    for (int i = 0; i < ROWS_PER_WARP; i++) {
      a[i].x += b[i].x;
      a[i].y += b[i].y;
      a[i].z += b[i].z;
      a[i].w += b[i].w;
      if (act) *at(mdst, i) = a[i];
      acc[i] = fmaf(l, dot4(a[i], pq), acc[i]);
    }
  }
  // open state: S = v phi(k)^T (new) or S += v phi(k)^T
  {
    float4 sv[ROWS_PER_WARP];
#pragma unroll
    for (int i = 0; i < ROWS_PER_WARP; i++) sv[i] = (open_new || !act) ? z4 : *at(open_slot, i);
    const float l = lam[open_slot];
#pragma unroll
    for (int i = 0; i < ROWS_PER_WARP; i++) {
      sv[i].x = fmaf(vr[i], pk[0], sv[i].x);
      sv[i].y = fmaf(vr[i], pk[1], sv[i].y);
      sv[i].z = fmaf(vr[i], pk[2], sv[i].z);
      sv[i].w = fmaf(vr[i], pk[3], sv[i].w);
      if (act) *at(open_slot, i) = sv[i];
      acc[i] = fmaf(l, dot4(sv[i], pq), acc[i]);
    }
  }
  // every other live state is read once (two slots in flight per lane)
  const int m = cc.m[u];
  const int32_t *order = cc.order + (size_t)u * C;
  int p = 0;
  for (; p + 1 < m; p += 2) {
    const int s0 = order[p], s1 = order[p + 1];
    const bool u0 = act && s0 != open_slot && s0 != mdst;
    const bool u1 = act && s1 != open_slot && s1 != mdst;
    float4 x0[ROWS_PER_WARP], x1[ROWS_PER_WARP];
#pragma unroll
    for (int i = 0; i < ROWS_PER_WARP; i++) {
      x0[i] = u0 ? __ldcs(at(s0, i)) : z4;
      x1[i] = u1 ? __ldcs(at(s1, i)) : z4;
    }
    const float l0 = u0 ? lam[s0] : 0.f, l1 = u1 ? lam[s1] : 0.f;
#pragma unroll
    for (int i = 0; i < ROWS_PER_WARP; i++) {
      acc[i] = fmaf(l0, dot4(x0[i], pq), acc[i]);
      acc[i] = fmaf(l1, dot4(x1[i], pq), acc[i]);
    }
  }
  for (; p < m; p++) {
    const int s0 = order[p];
    if (!act || s0 == open_slot || s0 == mdst) continue;
    const float l0 = lam[s0];
#pragma unroll
    for (int i = 0; i < ROWS_PER_WARP; i++) acc[i] = fmaf(l0, dot4(__ldcs(at(s0, i)), pq), acc[i]);
  }
#pragma unroll
  for (int i = 0; i < ROWS_PER_WARP; i++) {
    float sum = acc[i];
    for (int off = 16; off; off >>= 1) sum += __shfl_xor_sync(FULL, sum, off);
    if (lane == 0) store_out(o, dt, row + r0 + i, sum);
  }
}

}  // namespace

size_t decode_ws_bytes(int32_t N, int32_t H, int32_t C) {
  const size_t U = (size_t)N * H;
  return ((U * C * sizeof(float) + 255) / 256 * 256) + U * sizeof(int4) + 256;
}

cudaError_t launch_decode_decide(const dla_cache &cc, float tau, int32_t dt, const void *q,
                                 const void *k, void *ws, uint8_t *boundary, int32_t *merge_i,
                                 int32_t *dev_status, cudaStream_t s, const uint8_t *active) {
  const int U = cc.N * cc.H;
  DecodeWs w = carve_ws(ws, U, cc.C);
  k_decode_decide<<<(U + 3) / 4, 128, 0, s>>>(cc, tau, dt, q, k, w, boundary, merge_i,
                                              dev_status, active);
  return cudaGetLastError();
}

cudaError_t launch_decode_stream(const dla_cache &cc, int32_t dt, const void *q, const void *k,
                                 const void *v, void *o, void *ws, cudaStream_t s) {
  const int U = cc.N * cc.H;
  DecodeWs w = carve_ws(ws, U, cc.C);
  dim3 g((cc.d_k + ROWS_PER_CTA - 1) / ROWS_PER_CTA, U);
  switch (cc.d_k) {
    case 32: k_decode_stream<32><<<g, WARPS * 32, 0, s>>>(cc, dt, q, k, v, o, w); break;
    case 64: k_decode_stream<64><<<g, WARPS * 32, 0, s>>>(cc, dt, q, k, v, o, w); break;
    case 128: k_decode_stream<128><<<g, WARPS * 32, 0, s>>>(cc, dt, q, k, v, o, w); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

// ---- decode step without caller-provided scratch ---------------------------
// For callers that cannot allocate device memory themselves (see
// dla_decode_step_static in dla.h).  The scratch is one file-scope device
// array shared by every call on a device; the host resolves its device
// address with cudaGetSymbolAddress (the array's name is not a device pointer
// in host code).  The address belongs to the CUDA context the module was
// loaded in, so it is kept per device together with that context's id: after
// a cudaDeviceReset (or any other teardown) the next call on the device runs
// in a new context and looks the address up again.
namespace {
constexpr size_t STATIC_DECODE_BYTES = (size_t)8 << 20;
__device__ __align__(256) unsigned char g_decode_scratch[STATIC_DECODE_BYTES];
constexpr int MAX_DEVICES = 64;
std::mutex g_scratch_mu;
unsigned long long g_scratch_ctx[MAX_DEVICES];  // id of the context of g_scratch_addr
void *g_scratch_addr[MAX_DEVICES];

typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long *);

// Id of the calling thread's current context (false when none is current or
// the driver has no context ids).
bool current_ctx_id(unsigned long long *id) {
  static CtxGetCurrentFn get_cur = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static bool looked = false;
  if (!looked) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_cur = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
    looked = true;
  }
  CUcontext ctx = nullptr;
  if (!get_cur || !get_id || get_cur(&ctx) != CUDA_SUCCESS || !ctx) return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}

cudaError_t static_scratch(void **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= MAX_DEVICES) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  unsigned long long id = 0;
  if (current_ctx_id(&id) && g_scratch_addr[dev] && g_scratch_ctx[dev] == id) {
    *out = g_scratch_addr[dev];
    return cudaSuccess;
  }
  // first call on this device, or its context changed: resolve the address
  // (this also makes the device's primary context current)
  void *p = nullptr;
  e = cudaGetSymbolAddress(&p, g_decode_scratch);
  if (e != cudaSuccess) return e;
  if (current_ctx_id(&id)) {
    g_scratch_addr[dev] = p;
    g_scratch_ctx[dev] = id;
  } else {
    g_scratch_addr[dev] = nullptr;  // no context id: resolve on every call
  }
  *out = p;
  return cudaSuccess;
}
}  // namespace

size_t static_decode_max_bytes() { return STATIC_DECODE_BYTES; }

cudaError_t static_decode_scratch(void **out) { return static_scratch(out); }

}  // namespace dla
