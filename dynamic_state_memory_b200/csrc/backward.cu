// backward.cu -- gradient of a prefill's output with respect to q, k and v at
// the decisions the prefill took (dla_prefill_backward).
//
// Dynamic Linear Attention | Chlience Paper Archive, section 5.1 (states),
// 5.2 (merges), 5.3 (readout): the boundaries and merges are piecewise
// constant in the keys, so wherever the forward is differentiable its
// gradient is the one with the decision trace held fixed.  With the trace
// fixed, every token s <= t lies in exactly one live state at time t (states
// are contiguous token ranges) and the readout is a masked attention
//   o_t = sum_{s <= t} lambda_{t, i(s,t)} (phi(q_t) . phi(k_s)) v_s,
//   lambda_{t, .} = softmax_i(phi(q_t) . mu_i / sqrt(d)), mu_i the mean of
//   phi(k) over state i's tokens at time t.
// With P = phi(q_t) . phi(k_s) and dA = dO_t . v_s:
//   dlambda_i = sum_{s in state i} dA P,
//   da_i      = lambda_i (dlambda_i - sum_j lambda_j dlambda_j),
//   c[t, s]   = dA lambda_{i(s,t)} + da_{i(s,t)} / (sqrt(d) n_{i(s,t)}),
//   dphi(q_t) = sum_s c[t, s] phi(k_s),  dphi(k_s) = sum_t c[t, s] phi(q_t),
//   dv_s      = sum_t lambda_{t, i(s,t)} P[t, s] dO_t,
// then through phi' (1 for x > 0, e^x otherwise).
//
// Three kernels, all SIMT and quadratic in T (a first, exact path):
//   k_bw_prep  one CTA per stream: phi(q), phi(k) in fp32, fp64 prefix sums of
//              phi(k) (the means), and, walking the trace, the live states'
//              first tokens after every token's decision;
//   k_bw_rows  one CTA per (stream, t): lambda, dlambda, da, dphi(q_t), and
//              the per-state lambda and da / (sqrt(d) n) for the next kernel;
//   k_bw_cols  one CTA per (stream, s): dv_s and dphi(k_s).
#include "dla_internal.cuh"

namespace dla {
namespace {

constexpr int BW_THREADS = 128;
constexpr int BW_TMAX = 4096;  // two fp32 arrays of T entries in shared memory
constexpr int BW_CMAX = 128;

struct BwWs {
  float *fq, *fk;   // [heads][T][d] phi(q), phi(k)
  double *zp;       // [heads][T + 1][d] prefix sums of phi(k) (fp64)
  int32_t *starts;  // [heads][T][C] first token of each live state after token t
  int32_t *mt;      // [heads][T] live states after token t
  float *lam;       // [heads][T][C] lambda_{t, i}
  float *ecoef;     // [heads][T][C] da_{t, i} / (sqrt(d) n_i)
};

size_t al256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

size_t bw_layout(int64_t heads, int64_t T, int64_t d, int64_t C, BwWs *w, uint8_t *base) {
  size_t off = 0;
  auto take = [&](size_t bytes) -> uint8_t * {
    uint8_t *p = base ? base + off : nullptr;
    off += al256(bytes);
    return p;
  };
  BwWs l;
  l.fq = reinterpret_cast<float *>(take(sizeof(float) * heads * T * d));
  l.fk = reinterpret_cast<float *>(take(sizeof(float) * heads * T * d));
  l.zp = reinterpret_cast<double *>(take(sizeof(double) * heads * (T + 1) * d));
  l.starts = reinterpret_cast<int32_t *>(take(sizeof(int32_t) * heads * T * C));
  l.mt = reinterpret_cast<int32_t *>(take(sizeof(int32_t) * heads * T));
  l.lam = reinterpret_cast<float *>(take(sizeof(float) * heads * T * C));
  l.ecoef = reinterpret_cast<float *>(take(sizeof(float) * heads * T * C));
  if (w) *w = l;
  return off;
}

struct BwArgs {
  const void *q, *k, *v, *dO;
  int32_t dtype, T, d, C;
  dla_trace trace;
  float *dq, *dk, *dv;
  int32_t *dev_status;
};

__device__ __forceinline__ float dphi32(float x) { return x > 0.f ? 1.f : expf(x); }

__device__ __forceinline__ float warp_sum_f(float x) {
#pragma unroll
  for (int off = 16; off; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
  return x;
}

// ---- per stream: phi operands, prefix sums, live-state table ---------------
__global__ void __launch_bounds__(BW_THREADS) k_bw_prep(BwArgs a, BwWs w) {
  const int u = blockIdx.x, tid = threadIdx.x, lane = tid & 31;
  const int T = a.T, d = a.d, C = a.C;
  const size_t row0 = (size_t)u * T * d;
  for (int e = tid; e < T * d; e += BW_THREADS) {
    w.fq[row0 + e] = phi32(load_in(a.q, a.dtype, row0 + e));
    w.fk[row0 + e] = phi32(load_in(a.k, a.dtype, row0 + e));
  }
  if (tid < d) {  // the means' sums in fp64, token order
    double *zp = w.zp + (size_t)u * (T + 1) * d + tid;
    double acc = 0.0;
    zp[0] = 0.0;
    for (int t = 0; t < T; t++) {
      acc += phi64((double)load_in(a.k, a.dtype, row0 + (size_t)t * d + tid));
      zp[(size_t)(t + 1) * d] = acc;
    }
  }
  if (tid >= 32) return;
  // warp 0: the live states' first tokens after each token's decision
  __shared__ int st[BW_CMAX];
  const uint8_t *bnd = a.trace.boundary + (size_t)u * T;
  const int cap = a.trace.cap;
  int cnt = a.trace.merge_count[u];
  if (cnt > cap) {
    if (lane == 0) set_status(a.dev_status, DLA_ERR_TRACE_OVERFLOW);
    cnt = cap;
  }
  const int32_t *mt_ = a.trace.merge_t + (size_t)u * cap;
  const int32_t *mi_ = a.trace.merge_i + (size_t)u * cap;
  int m = 0, mp = 0;
  bool bad = false;
  for (int t = 0; t < T; t++) {
    if (bnd[t]) {
      if (mp < cnt && mt_[mp] == t) {
        const int r = mi_[mp] + 1;  // the merged pair's right member goes
        if (r < 1 || r >= m) {
          bad = true;
        } else {
          int tmp[BW_CMAX / 32];
#pragma unroll
          for (int q = 0; q < BW_CMAX / 32; q++) {
            const int j = lane + 32 * q;
            tmp[q] = (j >= r && j + 1 < m) ? st[j + 1] : 0;
          }
          __syncwarp();
#pragma unroll
          for (int q = 0; q < BW_CMAX / 32; q++) {
            const int j = lane + 32 * q;
            if (j >= r && j + 1 < m) st[j] = tmp[q];
          }
          m--;
        }
        mp++;
      }
      if (m >= C) {
        bad = true;
      } else {
        if (lane == 0) st[m] = t;
        m++;
      }
      __syncwarp();
    }
    if (m == 0) bad = true;  // token 0 of an empty cache opens a state
    int32_t *dst = w.starts + ((size_t)u * T + t) * C;
    for (int i = lane; i < m; i += 32) dst[i] = st[i];
    if (lane == 0) w.mt[(size_t)u * T + t] = m;
    __syncwarp();
  }
  if (mp != cnt) bad = true;  // a merge that falls on no boundary
  if (bad && lane == 0) set_status(a.dev_status, DLA_ERR_INVALID_ARG);
}

// ---- per (stream, t): softmax, its gradient, dphi(q_t) ---------------------
__global__ void __launch_bounds__(BW_THREADS) k_bw_rows(BwArgs a, BwWs w) {
  extern __shared__ float s_dyn[];  // [2][T]: dA (then c), P
  __shared__ float s_fq[128], s_do[128];
  __shared__ int s_st[BW_CMAX + 1];
  __shared__ float s_lam[BW_CMAX], s_e[BW_CMAX];
  __shared__ double s_red[BW_THREADS / 32];
  const int u = blockIdx.y, t = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int T = a.T, d = a.d, C = a.C;
  float *s_dA = s_dyn, *s_P = s_dyn + T;
  const size_t row = ((size_t)u * T + t) * d;
  int m = w.mt[(size_t)u * T + t];
  m = m < 1 ? 1 : (m > C ? C : m);  // (a bad trace is reported by k_bw_prep)
  if (tid < d) {
    s_fq[tid] = w.fq[row + tid];
    s_do[tid] = load_in(a.dO, a.dtype, row + tid);
  }
  for (int i = tid; i < m; i += BW_THREADS) {
    int s0 = w.starts[((size_t)u * T + t) * C + i];
    s_st[i] = s0 < 0 ? 0 : (s0 > t ? t : s0);
  }
  if (tid == 0) s_st[m] = t + 1;
  __syncthreads();
  // logits a_i = phi(q_t) . mu_i / sqrt(d) in fp64 (thread i: state i)
  const double rsd = 1.0 / sqrt((double)d);
  double ai = -INFINITY;
  int ni = 1;
  if (tid < m) {
    const int s0 = s_st[tid], s1 = s_st[tid + 1];
    ni = s1 - s0 > 0 ? s1 - s0 : 1;
    const double *z0 = w.zp + ((size_t)u * (T + 1) + s0) * d;
    const double *z1 = w.zp + ((size_t)u * (T + 1) + s1) * d;
    double acc = 0.0;
    for (int c = 0; c < d; c++) acc += (double)s_fq[c] * (z1[c] - z0[c]);
    ai = acc / ni * rsd;
  }
  auto block_max = [&](double x) -> double {
#pragma unroll
    for (int off = 16; off; off >>= 1) x = fmax(x, __shfl_xor_sync(0xffffffffu, x, off));
    if (lane == 0) s_red[warp] = x;
    __syncthreads();
    double r = s_red[0];
    for (int i = 1; i < BW_THREADS / 32; i++) r = fmax(r, s_red[i]);
    __syncthreads();
    return r;
  };
  auto block_sum = [&](double x) -> double {
#pragma unroll
    for (int off = 16; off; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
    if (lane == 0) s_red[warp] = x;
    __syncthreads();
    double r = 0.0;
    for (int i = 0; i < BW_THREADS / 32; i++) r += s_red[i];
    __syncthreads();
    return r;
  };
  const double amax = block_max(ai);
  const double ex = tid < m ? exp(ai - amax) : 0.0;
  const double lam = ex / block_sum(ex);
  // P and dA for every s <= t (a warp per s, lanes over the dimensions)
  for (int s = warp; s <= t; s += BW_THREADS / 32) {
    const size_t rs = ((size_t)u * T + s) * d;
    float p = 0.f, da = 0.f;
    for (int c = lane; c < d; c += 32) {
      p += s_fq[c] * w.fk[rs + c];
      da += s_do[c] * load_in(a.v, a.dtype, rs + c);
    }
    p = warp_sum_f(p);
    da = warp_sum_f(da);
    if (lane == 0) {
      s_P[s] = p;
      s_dA[s] = da;
    }
  }
  __syncthreads();
  // dlambda_i over state i's tokens, then the softmax's gradient
  double dl = 0.0;
  if (tid < m)
    for (int s = s_st[tid]; s < s_st[tid + 1]; s++) dl += (double)s_dA[s] * s_P[s];
  const double lsum = block_sum(tid < m ? lam * dl : 0.0);
  if (tid < m) {
    const double da = lam * (dl - lsum);
    const float e = (float)(da * rsd / ni);
    s_lam[tid] = (float)lam;
    s_e[tid] = e;
    w.lam[((size_t)u * T + t) * C + tid] = (float)lam;
    w.ecoef[((size_t)u * T + t) * C + tid] = e;
  }
  __syncthreads();
  // c[t, s] = dA lambda_i + e_i with i the state holding s (binary search)
  for (int s = tid; s <= t; s += BW_THREADS) {
    int lo = 0, hi = m - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_st[mid] <= s) lo = mid;
      else hi = mid - 1;
    }
    s_dA[s] = s_dA[s] * s_lam[lo] + s_e[lo];
  }
  __syncthreads();
  if (tid < d) {
    float g = 0.f;
    const float *fk = w.fk + (size_t)u * T * d + tid;
    for (int s = 0; s <= t; s++) g += s_dA[s] * fk[(size_t)s * d];
    a.dq[row + tid] = g * dphi32(load_in(a.q, a.dtype, row + tid));
  }
}

// ---- per (stream, s): dv_s and dphi(k_s) -----------------------------------
__global__ void __launch_bounds__(BW_THREADS) k_bw_cols(BwArgs a, BwWs w) {
  extern __shared__ float s_dyn[];  // [2][T - s]: lambda P, c
  __shared__ float s_fk[128], s_v[128];
  const int u = blockIdx.y, s = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int T = a.T, d = a.d, C = a.C;
  const int n = T - s;
  float *s_a = s_dyn, *s_c = s_dyn + n;
  const size_t row = ((size_t)u * T + s) * d;
  if (tid < d) {
    s_fk[tid] = w.fk[row + tid];
    s_v[tid] = load_in(a.v, a.dtype, row + tid);
  }
  __syncthreads();
  for (int t = s + warp; t < T; t += BW_THREADS / 32) {
    const size_t rt = ((size_t)u * T + t) * d;
    float p = 0.f, da = 0.f;
    for (int c = lane; c < d; c += 32) {
      p += w.fq[rt + c] * s_fk[c];
      da += load_in(a.dO, a.dtype, rt + c) * s_v[c];
    }
    p = warp_sum_f(p);
    da = warp_sum_f(da);
    if (lane == 0) {
      // the state holding s at time t: the last live state starting at or before s
      int m = w.mt[(size_t)u * T + t];
      m = m < 1 ? 1 : (m > C ? C : m);
      const int32_t *st = w.starts + ((size_t)u * T + t) * C;
      int lo = 0, hi = m - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (st[mid] <= s) lo = mid;
        else hi = mid - 1;
      }
      const float lam = w.lam[((size_t)u * T + t) * C + lo];
      s_a[t - s] = lam * p;
      s_c[t - s] = da * lam + w.ecoef[((size_t)u * T + t) * C + lo];
    }
  }
  __syncthreads();
  if (tid < d) {
    float gv = 0.f, gk = 0.f;
    for (int t = s; t < T; t++) {
      const size_t rt = ((size_t)u * T + t) * d + tid;
      gv += s_a[t - s] * load_in(a.dO, a.dtype, rt);
      gk += s_c[t - s] * w.fq[rt];
    }
    a.dv[row + tid] = gv;
    a.dk[row + tid] = gk * dphi32(load_in(a.k, a.dtype, row + tid));
  }
}

bool bw_shape_ok(const dla_config *c) {
  return c && c->B > 0 && c->H > 0 && c->T >= 0 && c->T <= BW_TMAX && c->d_k == c->d_v &&
         (c->d_k == 32 || c->d_k == 64 || c->d_k == 128) && c->C >= 2 && c->C <= BW_CMAX &&
         (c->in_dtype == DLA_F32 || c->in_dtype == DLA_BF16);
}

}  // namespace
}  // namespace dla

extern "C" {

size_t dla_backward_workspace_bytes(const dla_config *cfg) {
  if (!dla::bw_shape_ok(cfg)) return 0;
  return dla::bw_layout((int64_t)cfg->B * cfg->H, cfg->T, cfg->d_k, cfg->C, nullptr, nullptr);
}

dla_status dla_prefill_backward(const dla_config *cfg, const void *q, const void *k, const void *v,
                                const void *d_o, const dla_trace *trace, float *dq, float *dk,
                                float *dv, void *ws, size_t ws_bytes, int32_t *dev_status,
                                void *stream) {
  using namespace dla;
  if (!bw_shape_ok(cfg)) return cfg ? DLA_ERR_UNSUPPORTED : DLA_ERR_INVALID_ARG;
  if (!q || !k || !v || !d_o || !dq || !dk || !dv || !trace || !dev_status)
    return DLA_ERR_INVALID_ARG;
  if (!trace->boundary || !trace->merge_count || trace->cap < 0 ||
      (trace->cap > 0 && (!trace->merge_t || !trace->merge_i)))
    return DLA_ERR_INVALID_ARG;
  if (cfg->T == 0) return DLA_OK;
  const int64_t heads = (int64_t)cfg->B * cfg->H;
  BwWs w;
  const size_t need = bw_layout(heads, cfg->T, cfg->d_k, cfg->C, &w, static_cast<uint8_t *>(ws));
  if (!ws || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255)) return DLA_ERR_WORKSPACE;
  if (heads > 65535) return DLA_ERR_UNSUPPORTED;
  BwArgs a;
  a.q = q;
  a.k = k;
  a.v = v;
  a.dO = d_o;
  a.dtype = cfg->in_dtype;
  a.T = cfg->T;
  a.d = cfg->d_k;
  a.C = cfg->C;
  a.trace = *trace;
  a.dq = dq;
  a.dk = dk;
  a.dv = dv;
  a.dev_status = dev_status;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  k_bw_prep<<<(unsigned)heads, BW_THREADS, 0, s>>>(a, w);
  if (cudaGetLastError() != cudaSuccess) return DLA_ERR_CUDA;
  const dim3 g((unsigned)cfg->T, (unsigned)heads);
  const size_t smem = 2 * sizeof(float) * cfg->T;
  k_bw_rows<<<g, BW_THREADS, smem, s>>>(a, w);
  if (cudaGetLastError() != cudaSuccess) return DLA_ERR_CUDA;
  k_bw_cols<<<g, BW_THREADS, smem, s>>>(a, w);
  if (cudaGetLastError() != cudaSuccess) return DLA_ERR_CUDA;
  return DLA_OK;
}

}  // extern "C"
