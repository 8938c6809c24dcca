// fenwick.cu -- plan and states of the fixed Fenwick-bucket policy
// (Dynamic Linear Attention | Chlience Paper Archive, section 2 and section
// 5.4: Log-Linear Attention keeps O(log T) buckets; token t reads one block of
// size 2^b of [0, t-1] per set bit b of t, plus {t}).
//
// The structure does not depend on the data, so it is planned in parallel:
//   - a readout tile starts at T0 = c * M (M a power of two), so the blocks of
//     [0, T0 - 1] are whole-tile dyadic ranges: one tree node per set bit of c;
//   - leaves: per tile, the state sum S = sum v phi(k)^T, z = sum phi(k)
//     (on the tensor cores for bf16 d = 128, else k_fen_leaves);
//   - k_fen_means: every node's phi(k) sum and count (children added level by
//   level, one block per head), so the readout's prologue can start while the
//   states are still being summed;
//   - k_fen_sub: node states four levels at a time.  A CTA takes 16 nodes of
//   the pass's base level and a slice of their elements, and adds them in
//   order with a binary counter of partial sums in registers, so every node
//   of the four levels above is formed once (left child + right child) and
//   only the subtree roots, the next pass's base, are stored in fp32;
//   even-indexed nodes are written as frozen versions (fp32 or the bf16 UMMA
//   layout).  A block of size 2^b in a prefix [0, T0) starts at a multiple
//   of 2^(b+1), so only even-indexed nodes are ever atoms; odd ones only
//   build their parents;
//   - k_fen_plan: per tile, the atoms (tree nodes, oldest first) and the
//     in-tile events: every token is a boundary, and at offset o >= 1 the
//     binary-counter carry merges the two newest blocks (trailing ones of
//     o - 1) times; those blocks are always in-tile pieces.
// The readout kernels are the same as for the DLA policy.
#include "dla_internal.cuh"
#include "tc_ptx.cuh"

namespace dla {
namespace {

constexpr int THREADS = 256;

struct FenTree {
  float *S;    // [heads][nodes][D][D] fp32
  float *z;    // [heads][nodes][D]
  int32_t nodes;
  int32_t levels;       // leaves are level 0
  int32_t off[24];      // first node of each level
};

// node id of (level, index)
__device__ __forceinline__ int node_id(const FenTree &tr, int level, int index) {
  return tr.off[level] + index;
}

// The frozen version of node v (all threads of the block): the state, and
// with `means` its phi(k) sum and count.
template <int D>
__device__ void write_version(const Dims &dm, const Plan &pl, int u, int v, const float *S,
                              const float *z, float n, bool bf16, bool means = true) {
  // S: fp32 [D][D] in global memory
  if (bf16) {
    uint8_t *Vd = static_cast<uint8_t *>(pl.ver_S) + ((size_t)u * dm.vmax + v) * D * D * 2;
    for (int ch = threadIdx.x; ch < D * D / 8; ch += THREADS) {
      const int r = (ch * 8) / D, c0 = (ch * 8) % D;
      const float *src = S + (size_t)r * D + c0;
      *reinterpret_cast<uint4 *>(Vd + tc::sw128_offset(r, c0, D)) =
          make_uint4(tc::pack_bf16(src[0], src[1]), tc::pack_bf16(src[2], src[3]),
                     tc::pack_bf16(src[4], src[5]), tc::pack_bf16(src[6], src[7]));
    }
  } else {
    float *Vd = static_cast<float *>(pl.ver_S) + ((size_t)u * dm.vmax + v) * D * D;
    for (int e = threadIdx.x; e < D * D; e += THREADS) Vd[e] = S[e];
  }
  if (!means) return;
  for (int c = threadIdx.x; c < D; c += THREADS) pl.ver_z[((size_t)u * dm.vmax + v) * D + c] = z[c];
  if (threadIdx.x == 0) pl.ver_n[(size_t)u * dm.vmax + v] = n;
}

// Leaves: per (head, tile) the tile's full state sum (only tiles that are
// blocks of some later tile start are needed, i.e. tiles c < ntiles - 1).
template <int D>
__global__ void __launch_bounds__(THREADS) k_fen_leaves(Dims dm, Plan pl, CallArgs ca, FenTree tr,
                                                        int ntiles, bool bf16) {
  constexpr int PER = D * D / THREADS;
  const int u = blockIdx.y, c = blockIdx.x;
  if (c >= ntiles) return;
  const int M = dm.M;
  const int T0 = c * M, len = min(M, dm.T - T0);
  __shared__ float s_k[32][D];
  __shared__ float s_v[32][D];
  float acc[PER];
#pragma unroll
  for (int i = 0; i < PER; i++) acc[i] = 0.f;
  float zacc = 0.f;
  const int e0 = threadIdx.x * PER;  // consecutive elements of one row
  const int r = e0 / D, c0 = e0 % D;
  const size_t row0 = (size_t)u * dm.T + T0;
  for (int s0 = 0; s0 < len; s0 += 32) {
    const int nt = min(32, len - s0);
    __syncthreads();
    for (int e = threadIdx.x; e < 32 * D; e += THREADS) {
      const int s = e / D, cc = e % D;
      const bool ok = s < nt;
      s_k[s][cc] = ok ? phi32(load_in(ca.k, ca.in_dtype, (row0 + s0 + s) * D + cc)) : 0.f;
      s_v[s][cc] = ok ? load_in(ca.v, ca.in_dtype, (row0 + s0 + s) * D + cc) : 0.f;
    }
    __syncthreads();
    for (int s = 0; s < nt; s++) {
      const float vv = s_v[s][r];
#pragma unroll
      for (int i = 0; i < PER; i++) acc[i] = fmaf(vv, s_k[s][c0 + i], acc[i]);
      if (threadIdx.x < D) zacc += s_k[s][threadIdx.x];
    }
  }
  const int nid = node_id(tr, 0, c);
  float *S = tr.S + ((size_t)u * tr.nodes + nid) * D * D;
#pragma unroll
  for (int i = 0; i < PER; i++) S[e0 + i] = acc[i];
  float *z = tr.z + ((size_t)u * tr.nodes + nid) * D;
  if (threadIdx.x < D) z[threadIdx.x] = zacc;
  __syncthreads();
  write_version<D>(dm, pl, u, nid, S, z, (float)len, bf16);
}

// phi(k) sums and counts of every node above the leaves (one block per head,
// level by level): z(l, i) = z(l-1, 2i) + z(l-1, 2i+1), also as version means.
template <int D>
__global__ void __launch_bounds__(THREADS) k_fen_means(Dims dm, Plan pl, FenTree tr, int ntiles) {
  const int u = blockIdx.x;
  for (int l = 1; l < tr.levels; l++) {
    const int count = ntiles >> l;
    __syncthreads();  // level l - 1 is complete
    for (int e = threadIdx.x; e < count * D; e += THREADS) {
      const int i = e / D, c = e % D;
      const int a = node_id(tr, l - 1, 2 * i), b = node_id(tr, l - 1, 2 * i + 1);
      const int nid = node_id(tr, l, i);
      const float z = tr.z[((size_t)u * tr.nodes + a) * D + c] + tr.z[((size_t)u * tr.nodes + b) * D + c];
      tr.z[((size_t)u * tr.nodes + nid) * D + c] = z;
      pl.ver_z[((size_t)u * dm.vmax + nid) * D + c] = z;
      if (c == 0) pl.ver_n[(size_t)u * dm.vmax + nid] = (float)(dm.M << l);
    }
  }
}

// Levels base + 1 .. base + SUBL of the tree, from the (stored) nodes of level
// `base`: block (x, head) takes subtree x / nslice (SUBN consecutive base
// nodes) and element slice x % nslice of SUB_EPT * SUB_THREADS elements;
// thread i holds SUB_EPT consecutive elements of one row of each state.
constexpr int SUBL = 4, SUBN = 1 << SUBL;
constexpr int SUB_THREADS = 256, SUB_EPT = 8;

template <int D>
__global__ void __launch_bounds__(SUB_THREADS) k_fen_sub(Dims dm, Plan pl, FenTree tr, int base,
                                                         int nbase, int nslice, bool bf16) {
  const int u = blockIdx.y;
  const int sub = blockIdx.x / nslice, slice = blockIdx.x % nslice;
  const int e0 = (slice * SUB_THREADS + threadIdx.x) * SUB_EPT;  // first element of the thread
  if (e0 >= D * D) return;
  const int r = e0 / D, c0 = e0 % D;
  float acc[SUBL][SUB_EPT];  // pending left child of each level above the base
  const int first = sub * SUBN;
  const int last = min(first + SUBN, nbase);
  for (int j = first; j < last; j++) {
    float x[SUB_EPT];
    const float *src = tr.S + ((size_t)u * tr.nodes + node_id(tr, base, j)) * D * D + e0;
#pragma unroll
    for (int i = 0; i < SUB_EPT; i += 4) {
      const float4 v = *reinterpret_cast<const float4 *>(src + i);
      x[i] = v.x;
      x[i + 1] = v.y;
      x[i + 2] = v.z;
      x[i + 3] = v.w;
    }
    // carry: node j closes the node above it at every level where its index
    // (relative to the subtree) is odd, up to the first even one, where it
    // waits as a left child
    const int rel = j - first;
    bool carry = true;
#pragma unroll
    for (int l = 0; l < SUBL; l++) {
      if (carry) {
        if ((rel >> l) & 1) {
#pragma unroll
          for (int i = 0; i < SUB_EPT; i++) x[i] = acc[l][i] + x[i];
          const int level = base + l + 1;
          const int index = j >> (l + 1);  // the node's index at that level
          const int nid = node_id(tr, level, index);
          if (l + 1 == SUBL) {  // a subtree root: the next pass's base, in fp32
            float *dst = tr.S + ((size_t)u * tr.nodes + nid) * D * D + e0;
#pragma unroll
            for (int i = 0; i < SUB_EPT; i += 4)
              *reinterpret_cast<float4 *>(dst + i) = make_float4(x[i], x[i + 1], x[i + 2], x[i + 3]);
          }
          if ((index & 1) == 0) {  // an atom: its frozen version
            if (bf16) {
              uint8_t *Vd = static_cast<uint8_t *>(pl.ver_S) + ((size_t)u * dm.vmax + nid) * D * D * 2;
              *reinterpret_cast<uint4 *>(Vd + tc::sw128_offset(r, c0, D)) =
                  make_uint4(tc::pack_bf16(x[0], x[1]), tc::pack_bf16(x[2], x[3]),
                             tc::pack_bf16(x[4], x[5]), tc::pack_bf16(x[6], x[7]));
            } else {
              float *Vd = static_cast<float *>(pl.ver_S) + ((size_t)u * dm.vmax + nid) * D * D + e0;
#pragma unroll
              for (int i = 0; i < SUB_EPT; i += 4)
                *reinterpret_cast<float4 *>(Vd + i) = make_float4(x[i], x[i + 1], x[i + 2], x[i + 3]);
            }
          }
        } else {
#pragma unroll
          for (int i = 0; i < SUB_EPT; i++) acc[l][i] = x[i];
          carry = false;
        }
      }
    }
  }
}

// Per (head, tile): atoms = tree nodes of the blocks of [0, T0-1], events.
__global__ void k_fen_plan(Dims dm, Plan pl, FenTree tr, int ntiles) {
  const int u = blockIdx.y;
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= ntiles) return;
  const int M = dm.M;
  const int T0 = c * M, len = min(M, dm.T - T0);
  int m0 = 0;
  int start = 0;  // in tiles
  for (int b = 30; b >= 0; b--) {
    if ((c >> b) & 1) {
      pl.tile_atoms[((size_t)u * dm.tiles + c) * dm.amax + m0] = node_id(tr, b, start >> b);
      m0++;
      start += 1 << b;
    }
  }
  pl.tile_m0[(size_t)u * dm.tiles + c] = m0;
  pl.tile_nev[(size_t)u * dm.tiles + c] = len;
  for (int o = 0; o < len; o++) {
    pl.tile_ev_off[((size_t)u * dm.tiles + c) * M + o] = o;
    int code = EV_NO_MERGE;
    if (o >= 1) {
      const int ones = __ffs(~(o - 1)) - 1;  // trailing ones of o - 1
      if (ones > 0) code = -(ones + 1);
    }
    pl.tile_ev_mrg[((size_t)u * dm.tiles + c) * M + o] = code;
  }
}

// Plan, leaves and every node's means (what the readout's prologue needs),
// then (levels == true) the node states and versions.
template <int D>
cudaError_t run_d(const Dims &dm, const Plan &pl, const CallArgs &ca, const FenTree &tr,
                  int ntiles, bool bf16, bool levels, cudaStream_t s) {
  if (levels) {
    // four levels per launch, from the leaves up
    const int nslice = (D * D + SUB_THREADS * SUB_EPT - 1) / (SUB_THREADS * SUB_EPT);
    for (int base = 0; base + 1 < tr.levels; base += SUBL) {
      const int nbase = ntiles >> base;
      if (nbase < 2) break;
      const int nsub = (nbase + SUBN - 1) / SUBN;
      k_fen_sub<D><<<dim3(nsub * nslice, dm.heads), SUB_THREADS, 0, s>>>(dm, pl, tr, base, nbase,
                                                                        nslice, bf16);
    }
    return cudaGetLastError();
  }
  k_fen_plan<<<dim3((ntiles + 127) / 128, dm.heads), 128, 0, s>>>(dm, pl, tr, ntiles);
  if (bf16 && D == 128) {
    // leaves on the tensor cores (tile state sums, phi(k) sums, bf16 versions)
    const cudaError_t e = launch_fen_leaves_tc(dm, pl, ca, tr.S, tr.z, tr.nodes, ntiles, s);
    if (e != cudaSuccess) return e;
  } else {
    k_fen_leaves<D><<<dim3(ntiles, dm.heads), THREADS, 0, s>>>(dm, pl, ca, tr, ntiles, bf16);
  }
  if (tr.levels > 1) k_fen_means<D><<<dm.heads, THREADS, 0, s>>>(dm, pl, tr, ntiles);
  return cudaGetLastError();
}

}  // namespace

// Tree sizes for T tokens in tiles of M: number of nodes and levels.
void fen_tree_shape(int T, int M, int *nodes, int *levels) {
  const int ntiles = (T + M - 1) / M;
  int n = 0, l = 0;
  for (int cnt = ntiles; cnt > 0 && l < 24; cnt >>= 1, l++) n += cnt;
  *nodes = n > 0 ? n : 1;
  *levels = l > 0 ? l : 1;
}

cudaError_t launch_fenwick(const Dims &dm, const Plan &pl, const CallArgs &ca, float *treeS,
                           float *treeZ, bool bf16, bool levels, cudaStream_t s) {
  FenTree tr{};
  tr.S = treeS;
  tr.z = treeZ;
  const int ntiles = (dm.T + dm.M - 1) / dm.M;
  fen_tree_shape(dm.T, dm.M, &tr.nodes, &tr.levels);
  int off = 0;
  for (int l = 0; l < tr.levels; l++) {
    tr.off[l] = off;
    off += ntiles >> l;
  }
  switch (dm.D) {
    case 32: return run_d<32>(dm, pl, ca, tr, ntiles, bf16, levels, s);
    case 64: return run_d<64>(dm, pl, ca, tr, ntiles, bf16, levels, s);
    case 128: return run_d<128>(dm, pl, ca, tr, ntiles, bf16, levels, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace dla
