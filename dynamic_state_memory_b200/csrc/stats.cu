// stats.cu -- per-stream summary of a prefill's decision trace, on the device.
//
// What the pages suggest watching in a DLA memory (the Chlience page's list of
// what to observe: boundary counts, merge frequency, how many states are
// live), reduced from a dla_trace without copying it to the host.  The live
// count read by token t is
//   m_t = m_before + (boundaries at s <= t) - (merges at s <= t)
// (a boundary seals the open state and opens a new one, +1; a capacity merge
// joins two states, -1; both happen only at boundary tokens).  One block per
// stream walks the call's tokens in chunks: the merges of a chunk are
// scattered into a shared count per token, and a block scan of
// (boundary - merges) gives every m_t.
#include "dla_internal.cuh"

namespace dla {
namespace {

constexpr int ST_THREADS = 256;
constexpr int ST_CHUNK = 4096;  // tokens per shared-memory chunk

__global__ void __launch_bounds__(ST_THREADS) k_trace_stats(dla_trace tr, int T,
                                                             const int32_t *m_before,
                                                             const int64_t *t_before, int tile,
                                                             dla_stats out, int32_t *dev_status) {
  __shared__ int s_merge[ST_CHUNK];
  __shared__ long long s_wsum[ST_THREADS / 32];
  __shared__ int s_wmax[ST_THREADS / 32];
  __shared__ long long s_carry;
  const int u = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint8_t *b = tr.boundary + (size_t)u * T;
  const int32_t *mt = tr.merge_t + (size_t)u * tr.cap;
  int mc = tr.merge_count[u];
  if (mc > tr.cap) {  // the trace lost merges: the counts would be wrong
    if (tid == 0) set_status(dev_status, DLA_ERR_TRACE_OVERFLOW);
    mc = tr.cap;
  }
  const long long t0 = t_before ? t_before[u] : 0;
  if (tid == 0) s_carry = m_before ? m_before[u] : 0;
  long long live_sum = 0, atom_rows = 0;
  int live_max = 0, nb = 0;
  for (int c0 = 0; c0 < T; c0 += ST_CHUNK) {
    for (int i = tid; i < ST_CHUNK; i += ST_THREADS) s_merge[i] = 0;
    __syncthreads();
    for (int j = tid; j < mc; j += ST_THREADS) {
      const long long lt = (long long)mt[j] - t0 - c0;
      if (lt >= 0 && lt < ST_CHUNK) atomicAdd(&s_merge[lt], 1);
    }
    __syncthreads();
    for (int s0 = 0; s0 < ST_CHUNK && c0 + s0 < T; s0 += ST_THREADS) {
      const int t = c0 + s0 + tid;
      const int bt = t < T ? (int)b[t] : 0;
      int dlt = t < T ? bt - s_merge[s0 + tid] : 0;
      // inclusive block scan of the deltas
      int x = dlt;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, off);
        if (lane >= off) x += y;
      }
      if (lane == 31) s_wmax[warp] = x;  // warp totals (reused as scratch)
      __syncthreads();
      int before = 0, total = 0;
      for (int w = 0; w < ST_THREADS / 32; w++) {
        const int wt = s_wmax[w];
        if (w < warp) before += wt;
        total += wt;
      }
      const long long m = s_carry + before + x;  // states read by token t
      __syncthreads();
      if (t < T) {
        live_sum += m;
        live_max = max(live_max, (int)m);
        nb += bt;
        // the readout's atoms: tile c >= 1 reads the states live after token c * tile - 1
        if (tile > 0 && (t + 1) % tile == 0 && t + 1 < T)
          atom_rows += (long long)min(tile, T - (t + 1)) * m;
      }
      if (tid == ST_THREADS - 1) s_carry += total;
      __syncthreads();
    }
  }
  // block sums
  long long ls = live_sum, ar = atom_rows;
  int lm = live_max, bb = nb;
#pragma unroll
  for (int off = 16; off; off >>= 1) {
    ls += __shfl_xor_sync(0xffffffffu, ls, off);
    ar += __shfl_xor_sync(0xffffffffu, ar, off);
    lm = max(lm, __shfl_xor_sync(0xffffffffu, lm, off));
    bb += __shfl_xor_sync(0xffffffffu, bb, off);
  }
  __shared__ long long s_ar[ST_THREADS / 32];
  __shared__ int s_bb[ST_THREADS / 32];
  if (lane == 0) {
    s_wsum[warp] = ls;
    s_ar[warp] = ar;
    s_wmax[warp] = lm;
    s_bb[warp] = bb;
  }
  __syncthreads();
  if (tid == 0) {
    long long a = 0, c = 0;
    int mx = 0, nbt = 0;
    for (int w = 0; w < ST_THREADS / 32; w++) {
      a += s_wsum[w];
      c += s_ar[w];
      mx = max(mx, s_wmax[w]);
      nbt += s_bb[w];
    }
    if (out.boundaries) out.boundaries[u] = nbt;
    if (out.merges) out.merges[u] = tr.merge_count[u];
    if (out.live_sum) out.live_sum[u] = a;
    if (out.live_max) out.live_max[u] = mx;
    if (out.atom_rows) out.atom_rows[u] = c;
  }
}

}  // namespace

cudaError_t launch_trace_stats(const dla_trace &tr, int heads, int T, const int32_t *m_before,
                               const int64_t *t_before, int tile, const dla_stats &out,
                               int32_t *dev_status, cudaStream_t s) {
  k_trace_stats<<<heads, ST_THREADS, 0, s>>>(tr, T, m_before, t_before, tile, out, dev_status);
  return cudaGetLastError();
}

}  // namespace dla
