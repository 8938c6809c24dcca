// build_tc.cu -- tcgen05 chunked state builder.
//
// For every readout tile (128 tokens) and every piece of it (a maximal run of
// tokens between in-tile boundaries) of at least PIECE_MIN tokens, computes
//   dS_p = sum_{s in p} v_s phi(k_s)^T = V_p^T phi(K_p)        (d_v x d_k, fp32)
// (the per-token state of Dynamic Linear Attention | Chlience Paper Archive,
// section 5.1, summed over the piece) on the tensor cores: A = V^T and
// B = phi(K)^T are both read MN-major straight from the TMA-loaded tiles
// (128-byte swizzle), K = tokens in steps of 16.  Rows of the 16-token blocks
// that straddle the piece's ends are zeroed in a copy of that block.  The
// accumulator lives in TMEM; 4 warps (one TMEM lane = one row of d_v) write it
// to the piece buffer, which the materializer adds to the open state (op
// ADDP).  Shorter pieces stay SIMT adds in the materializer.
//
// The phi(k) tile, as it sits in shared memory (two 64-column halves of 128
// rows, 128-byte swizzle), is also stored to the plan: it is the readout
// prologue's phi(K) operand.
//
// Leaf mode (fixed Fenwick policy): the one piece is the whole tile and the
// result is the tree leaf of that tile: fp32 state and phi(k) sum, plus the
// frozen bf16 version (UMMA layout), its phi(k) sum and token count.
#include "dla_internal.cuh"
#include "tc_ptx.cuh"

namespace dla {
namespace {
using namespace tc;

constexpr int M = 128;
constexpr int D = 128;
constexpr int THREADS = 128;
constexpr int TILE_BYTES = M * D * 2;
constexpr int BLK = 2048;  // one 16-token block of one 64-column half

struct FenLeaves {
  float *treeS;  // [heads][nodes][D][D]; null: piece mode
  float *treeZ;  // [heads][nodes][D]
  int nodes;
};

struct Smem {
  uint8_t k[TILE_BYTES];     // phi(k), rows = tokens, MN-major for B
  uint8_t v[TILE_BYTES];     // v, rows = tokens, MN-major for A
  uint8_t edge[2][2][BLK];   // masked copies of the first / last block: [which][half]
  uint64_t bar_load, bar_mma;
  uint32_t tmem_base;
  int abort;
  int np;
  int pst[M + 1], pen[M + 1];
};

__global__ void __launch_bounds__(THREADS, 1)
    k_build_tc(const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
               Dims dm, Plan pl, CallArgs ca, FenLeaves fen) {
  extern __shared__ uint8_t raw[];
  Smem &sm = *reinterpret_cast<Smem *>((reinterpret_cast<uintptr_t>(raw) + 1023) &
                                       ~static_cast<uintptr_t>(1023));
  const int u = blockIdx.y, c = blockIdx.x;
  const int T0 = c * M;
  const int Tw = tw_of(ca, u);
  if (T0 >= Tw) return;
  const int tid = threadIdx.x, warp = tid >> 5;
  volatile int *abort = &sm.abort;
  const int len = min(M, Tw - T0);
  if (warp == 0) tmem_alloc(&sm.tmem_base, 128);
  if (tid == 0) {
    mbar_init(&sm.bar_load, 1);
    mbar_init(&sm.bar_mma, 1);
    fence_mbar_init();
    sm.abort = 0;
    if (fen.treeS) {
      sm.pst[0] = 0;
      sm.pen[0] = len;
      sm.np = 1;
    } else {
      // runs of the tile: it starts one, and every boundary flag after its
      // first token starts the next (the first token either continues the
      // open state or opens a new one; the run starts there either way)
      const uint8_t *bf = pl.b + (size_t)u * dm.W + T0;
      int np = 0;
      sm.pst[np++] = 0;
      for (int i = 1; i < len; i++)
        if (bf[i]) sm.pst[np++] = i;
      for (int p = 0; p < np; p++) sm.pen[p] = p + 1 < np ? sm.pst[p + 1] : len;
      sm.np = np;
    }
    mbar_expect_tx(&sm.bar_load, 2 * TILE_BYTES);
    const int row = ca.w0 + T0;
    for (int h = 0; h < 2; h++) {
      tma_load_3d(sm.k + h * (TILE_BYTES / 2), &tk, &sm.bar_load, h * 64, row, u);
      tma_load_3d(sm.v + h * (TILE_BYTES / 2), &tv, &sm.bar_load, h * 64, row, u);
    }
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = sm.tmem_base;
  mbar_wait(&sm.bar_load, 0, abort);
  if (fen.treeS) {
    // leaf phi(k) sum in token order, from the raw tile (thread = column)
    float z = 0.f;
    for (int r = 0; r < len; r++) {
      const uint16_t x = *reinterpret_cast<const uint16_t *>(sm.k + sw128_offset(r, tid, M));
      z += phi32(__uint_as_float((uint32_t)x << 16));
    }
    const size_t node = (size_t)u * fen.nodes + c;
    fen.treeZ[node * D + tid] = z;
    pl.ver_z[((size_t)u * dm.vmax + c) * D + tid] = z;
    if (tid == 0) pl.ver_n[(size_t)u * dm.vmax + c] = (float)len;
    __syncthreads();
  }
  for (int i = tid; i < TILE_BYTES / 16; i += THREADS) {
    uint4 *p = reinterpret_cast<uint4 *>(sm.k) + i;
    uint4 x = *p;
    uint32_t *w = reinterpret_cast<uint32_t *>(&x);
#pragma unroll
    for (int j = 0; j < 4; j++) w[j] = pack_bf16(phi_bf16op(bf16_lo(w[j])), phi_bf16op(bf16_hi(w[j])));
    *p = x;
  }
  fence_proxy_async();
  __syncthreads();
  if (tid == 0 && pl.phi_k) {  // sm.k is not written again
    bulk_store(static_cast<uint8_t *>(pl.phi_k) + ((size_t)u * dm.tiles + c) * TILE_BYTES, sm.k,
               TILE_BYTES);
    bulk_commit();
  }

  const int np = sm.np;
  const int pbase = fen.treeS ? c : c * PIECES_PER_TILE;
  float *pieces = fen.treeS ? fen.treeS + (size_t)u * fen.nodes * D * D
                            : pl.pieces + (size_t)u * dm.pmax * D * D;
  const uint32_t k_s = smem_u32(sm.k), v_s = smem_u32(sm.v);
  int id = pbase;
  int phase = 0;
  for (int p = 0; p < np; p++) {
    const int a = sm.pst[p], b = sm.pen[p];
    if (b - a < PIECE_MIN && !fen.treeS) continue;
    const int jb0 = a >> 4, jb1 = (b - 1) >> 4;
    // masked copies of the straddling blocks (whole 128-byte rows zeroed)
    const bool edge0 = (a & 15) != 0 || (jb0 == jb1 && (b & 15) != 0);
    const bool edge1 = jb1 != jb0 && (b & 15) != 0;
    for (int e = tid; e < 2 * 2 * (BLK / 16); e += THREADS) {
      const int which = e / (2 * (BLK / 16)), rem = e % (2 * (BLK / 16));
      const int half = rem / (BLK / 16), ch = rem % (BLK / 16);  // 16-byte chunk
      const int jb = which == 0 ? jb0 : jb1;
      if ((which == 0 && !edge0) || (which == 1 && !edge1)) continue;
      const int r = ch / 8;  // row (token) inside the block: 128 bytes = 8 chunks
      const int tok = jb * 16 + r;
      uint4 x = *reinterpret_cast<const uint4 *>(sm.v + half * (TILE_BYTES / 2) + jb * BLK + ch * 16);
      if (tok < a || tok >= b) x = make_uint4(0, 0, 0, 0);
      *reinterpret_cast<uint4 *>(sm.edge[which][half] + ch * 16) = x;
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      for (int j = jb0; j <= jb1; j++) {
        uint64_t adesc;
        if (j == jb0 && edge0)
          adesc = sdesc(smem_u32(sm.edge[0][0]), BLK, 1024);
        else if (j == jb1 && edge1)
          adesc = sdesc(smem_u32(sm.edge[1][0]), BLK, 1024);
        else
          adesc = sdesc(v_s + j * BLK, TILE_BYTES / 2, 1024);
        const uint64_t bdesc = sdesc(k_s + j * BLK, TILE_BYTES / 2, 1024);
        mma_bf16(tbase, adesc, bdesc, idesc_bf16(M, D, 1, 1), j > jb0);
      }
      mma_commit(&sm.bar_mma);
    }
    mbar_wait(&sm.bar_mma, phase, abort);
    phase ^= 1;
    tc_fence_after();
    // TMEM lane = row r of d_v; write the fp32 row to the piece buffer
    {
      const int r = 32 * warp + (tid & 31);
      const uint32_t trow = tbase + ((uint32_t)(32 * warp) << 16);
      float4 *dst = reinterpret_cast<float4 *>(pieces + ((size_t)id * D + r) * D);
      uint8_t *ver = fen.treeS ? static_cast<uint8_t *>(pl.ver_S) + ((size_t)u * dm.vmax + c) * D * D * 2
                               : nullptr;
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t x[32];
        DLA_TMEM_LD32(trow + c0, x);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 8; i++)
          dst[c0 / 4 + i] = make_float4(__uint_as_float(x[4 * i]), __uint_as_float(x[4 * i + 1]),
                                        __uint_as_float(x[4 * i + 2]), __uint_as_float(x[4 * i + 3]));
        if (ver) {
#pragma unroll
          for (int i = 0; i < 4; i++)
            *reinterpret_cast<uint4 *>(ver + sw128_offset(r, c0 + 8 * i, D)) =
                make_uint4(pack_bf16(__uint_as_float(x[8 * i]), __uint_as_float(x[8 * i + 1])),
                           pack_bf16(__uint_as_float(x[8 * i + 2]), __uint_as_float(x[8 * i + 3])),
                           pack_bf16(__uint_as_float(x[8 * i + 4]), __uint_as_float(x[8 * i + 5])),
                           pack_bf16(__uint_as_float(x[8 * i + 6]), __uint_as_float(x[8 * i + 7])));
        }
      }
    }
    tc_fence_before();
    __syncthreads();
    id++;
  }
  if (tid == 0 && pl.phi_k) bulk_wait_read();
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tbase, 128);
  }
  if (tid == 0 && sm.abort) set_status(ca.dev_status, DLA_ERR_TIMEOUT);
}

}  // namespace

bool make_bf16_map(CUtensorMap *m, const void *base, int T, int heads);

static cudaError_t launch_tc(const Dims &dm, const Plan &pl, const CallArgs &ca, FenLeaves fen,
                             int ntiles, cudaStream_t s) {
  if (dm.M != M || dm.D != D || ca.in_dtype != DLA_BF16) return cudaErrorInvalidValue;
  CUtensorMap tk, tv;
  if (!make_bf16_map(&tk, ca.k, dm.T, dm.heads) || !make_bf16_map(&tv, ca.v, dm.T, dm.heads))
    return cudaErrorInvalidValue;
  const size_t sb = sizeof(Smem) + 1024;
  cudaError_t e = cudaFuncSetAttribute(k_build_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sb);
  if (e != cudaSuccess) return e;
  k_build_tc<<<dim3(ntiles, dm.heads), THREADS, sb, s>>>(tk, tv, dm, pl, ca, fen);
  return cudaGetLastError();
}

cudaError_t launch_build_tc(const Dims &dm, const Plan &pl, const CallArgs &ca, cudaStream_t s) {
  return launch_tc(dm, pl, ca, FenLeaves{nullptr, nullptr, 0}, dm.tiles, s);
}

// Fixed-policy tree leaves of tiles [0, ntiles) (version id of a leaf = its tile).
cudaError_t launch_fen_leaves_tc(const Dims &dm, const Plan &pl, const CallArgs &ca, float *treeS,
                                 float *treeZ, int nodes, int ntiles, cudaStream_t s) {
  return launch_tc(dm, pl, ca, FenLeaves{treeS, treeZ, nodes}, ntiles, s);
}

}  // namespace dla
