// readout_tc.cu -- tcgen05 tensor-core readout of 128-token tiles (bf16
// inputs, fp32 accumulation, d_k = d_v = 128), in two kernels.
//
// Same arithmetic as the SIMT readout (see readout_simt.cu for the atom /
// piece / epoch formulation of o_t = sum_i lambda_{t,i} S_i phi(q_t) with
// lambda_{t,i} = softmax_i(phi(q_t) . mu_i / sqrt(d_k)); Dynamic Linear
// Attention | Chlience Paper Archive, section 5.3), mapped onto Blackwell.
//
// k_phi_tc writes phi(q) of the window as the bf16 operand (it needs only the
// input, so it runs beside the engine); the state builder stores the phi(k)
// tiles it forms for its own products.
// k_readout_pre needs only the plan's atom lists and means, not the frozen
// state versions, so it runs beside the materializer:
//   TMA (128B swizzle) loads the phi(q) and v tiles, a bulk copy the builder's
//   phi(k) tile.
//   tcgen05.mma (kind::f16, M = 128 tokens) computes into tensor memory:
//     A  = phi(Q) phi(K)^T               (128 x 128)   TMEM cols [256, 384)
//     LA = phi(Q) Mu^T                   (128 x m0)    TMEM cols [384, 512)
//   Four warps (one TMEM lane = one token row each) turn LA and the row sums
//   of A into softmax weights per atom / piece and write
//   P = W o A (causal) as the bf16 A operand of
//     O_intra = P V                                    TMEM cols [256, 384)
//   It stores the atom weights W[atom][row] and O_intra (fp32) to the plan.
// k_readout_tc then runs the pipelined loop over atoms, over a run of
// consecutive tiles per CTA: the epilogue warps start from O_intra and put
// phi(Q) into tensor memory; per atom alpha, a bulk copy brings the frozen
// bf16 state version (already in the UMMA K-major swizzled layout) into one
// of 5 shared stages, two threads issue P_alpha = phi(Q) S_alpha^T (even / odd
// atoms) into three TMEM buffers with phi(Q) read from tensor memory, and 8
// epilogue warps accumulate W_alpha(t) * P_alpha in registers while the next
// MMAs run.
// Every wait on an mbarrier is bounded; a timeout sets DLA_ERR_TIMEOUT.
#include "dla_internal.cuh"
#include "tc_ptx.cuh"

namespace dla {
namespace {
using namespace tc;

constexpr int M = 128;
constexpr int D = 128;
constexpr int NSV = 5;   // version stages of the atom loop
constexpr int THREADS = 384;      // atom loop
constexpr int PRE_THREADS = 256;  // per-tile prologue
constexpr int TILE_BYTES = M * D * 2;
constexpr uint32_t VER_BYTES = D * D * 2;
constexpr int BW = 8;  // epoch bitmask words: atoms + pieces <= 256
constexpr uint32_t COL_AI = 256;  // phi(Q) of the atom loop
constexpr int NPB = 3;  // TMEM P buffers: cols [0,128), [128,256) and [384,512)
__device__ __forceinline__ uint32_t pbuf_col(int b) { return b == 2 ? 384u : (uint32_t)b * 128u; }
// phi(Q) as the A operand of the atom MMAs, in tensor memory, in one of two
// regions (par, alternating by tile): elements [64h, 64h + 64) of a row in
// cols COL_AI + 32 par + 64h + [0, 32), two per column
__device__ __forceinline__ uint32_t qa_col(int kstep, int par) {
  return COL_AI + 32 * par + (kstep < 4 ? 8 * kstep : 64 + 8 * (kstep - 4));
}
constexpr float INV_SQRT_D = 0.08838834764831845f;
// Tensor memory of the prologue (256 columns, two CTAs per SM): A, then P in
// place (the bf16 A operand of P V, laid out like phi(Q) above), in cols
// [0, 128); LA, then O_intra, in cols [128, 256).
constexpr uint32_t PRE_A = 0, PRE_LA = 128, PRE_COLS = 256;
__device__ __forceinline__ uint32_t pa_col(int kstep) {
  return PRE_A + (kstep < 4 ? 8 * kstep : 64 + 8 * (kstep - 4));
}
// column of P's elements [s0, s0 + 2n) (s0 even, within one half of 64)
__device__ __forceinline__ uint32_t p_col(int s0) { return PRE_A + 64 * (s0 >> 6) + ((s0 & 63) >> 1); }

// ---- per-tile outputs of the prologue in the plan ----------------------------
// W: fp32 [g][amax][M].  O_intra: bf16 [g][2][8][M][8] -- column 64 h + 8 i + e
// of row t at ((h * 8 + i) * M + t) * 8 + e, so that a warp's 32 rows read or
// write 512 contiguous bytes (its rounding is far inside the bf16 output's
// tolerance; the atom loop accumulates in fp32).
__device__ __forceinline__ size_t pre_o_chunk(int t, int h, int i) { return (size_t)(h * 8 + i) * M + t; }

struct PreSmem {
  uint8_t kp[TILE_BYTES];  // phi(K), then the v tile
  uint8_t q[TILE_BYTES];   // phi(Q)
  uint8_t mu[TILE_BYTES];  // bf16 atom means in the 128-row UMMA layout (its second
                           // K-half is 16 KB after the first, whatever the atom count)
                           // q and mu, once the first MMAs have read them, hold the
                           // values of pieces PREG.. (fp32 [piece][row], 128 pieces)
  uint64_t bar_load, bar_mma, bar_v, bar_la;
  uint32_t tmem_base;
  int abort;
  int m0, np, len, cont;
  float nA[128];
  int atom[128];
  int pst[M + 1], pen[M + 1], pidx[M];
  uint32_t bits[(M + 1) * BW];
};


static_assert(offsetof(PreSmem, mu) == offsetof(PreSmem, q) + TILE_BYTES, "q, mu adjacent");

// Shared memory of the persistent atom loop: the phi(Q) landing buffer, NSV
// version stages and a ring of NWC weight chunks of WCH atoms.
constexpr int NWC = 2, WCH = 32;
struct Smem {
  uint8_t q[TILE_BYTES];  // phi(Q) of a tile, on its way to tensor memory
  uint8_t st[NSV][VER_BYTES];
  float w[NWC][WCH * M];  // W[atom][row] of WCH atoms per chunk
  uint64_t bar_load, bar_qa, bar_qs, full[NSV], empty[NSV], tfull[NPB], tempty[NPB], wfull[NWC],
      wempty[NWC];
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(Smem) + 1024 <= 227 * 1024, "atom loop shared memory");

__device__ __forceinline__ bool bit_of(const uint32_t *b, int i) { return (b[i >> 5] >> (i & 31)) & 1u; }

// pairwise sum / max of 32 values (depth 5: the terms are independent)
__device__ __forceinline__ float sum32(const float (&x)[32]) {
  float y[16];
#pragma unroll
  for (int j = 0; j < 16; j++) y[j] = x[j] + x[j + 16];
#pragma unroll
  for (int w = 8; w >= 1; w >>= 1)
#pragma unroll
    for (int j = 0; j < w; j++) y[j] += y[j + w];
  return y[0];
}
__device__ __forceinline__ float max32(const float (&x)[32]) {
  float y[16];
#pragma unroll
  for (int j = 0; j < 16; j++) y[j] = fmaxf(x[j], x[j + 16]);
#pragma unroll
  for (int w = 8; w >= 1; w >>= 1)
#pragma unroll
    for (int j = 0; j < w; j++) y[j] = fmaxf(y[j], y[j + w]);
  return y[0];
}

// phi(q) of the window's rows as the bf16 operand of the readout: phi_q
// [heads][W][D], rows [0, Tw) (16 bytes per thread and step).
__global__ void __launch_bounds__(256) k_phi_tc(Dims dm, Plan pl, CallArgs ca) {
  const size_t per_head = (size_t)ca.Tw * (D / 8);
  const size_t total = per_head * dm.heads;
  for (size_t i = (size_t)blockIdx.x * 256 + threadIdx.x; i < total; i += (size_t)gridDim.x * 256) {
    const size_t u = i / per_head, r = i - u * per_head;
    const uint4 *src = static_cast<const uint4 *>(ca.q) + (u * dm.T + ca.w0) * (D / 8) + r;
    uint4 *dst = static_cast<uint4 *>(pl.phi_q) + u * dm.W * (D / 8) + r;
    uint4 x = *src;
    uint32_t *w = reinterpret_cast<uint32_t *>(&x);
#pragma unroll
    for (int e = 0; e < 4; e++) w[e] = pack_bf16(phi_bf16op(bf16_lo(w[e])), phi_bf16op(bf16_hi(w[e])));
    *dst = x;
  }
}

__global__ void __launch_bounds__(PRE_THREADS, 2)
    k_readout_pre(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tv,
                  Dims dm, Plan pl, CallArgs ca) {
  extern __shared__ uint8_t raw[];
  PreSmem &sm = *reinterpret_cast<PreSmem *>((reinterpret_cast<uintptr_t>(raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int u = blockIdx.y, c = blockIdx.x;
  const int T0 = c * M;
  const int Tw = tw_of(ca, u);
  if (T0 >= Tw) return;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  volatile int *abort = &sm.abort;
  const size_t g = (size_t)u * dm.tiles + c;  // tile index in the plan
  float *const preW = pl.pre_w + g * dm.amax * M;
  uint8_t *const mu_buf = sm.mu;

  // ---- setup: TMEM, barriers, tile loads first, then tile metadata --------
  if (warp == 1) tmem_alloc(&sm.tmem_base, PRE_COLS);
  if (tid == 0) {
    mbar_init(&sm.bar_load, 1);
    fence_mbar_init();
    mbar_expect_tx(&sm.bar_load, 2 * TILE_BYTES);
    for (int h = 0; h < 2; h++)
      tma_load_3d(sm.q + h * (TILE_BYTES / 2), &tq, &sm.bar_load, h * 64, T0, u);
    bulk_load(sm.kp, static_cast<const uint8_t *>(pl.phi_k) + g * TILE_BYTES, TILE_BYTES, &sm.bar_load);
  }
  const int m0 = pl.tile_m0[(size_t)u * dm.tiles + c];
  const int32_t *const atoms_g = pl.tile_atoms + ((size_t)u * dm.tiles + c) * dm.amax;
  const int m0c = min(m0, 128);  // atoms of the first logit chunk (all of them unless unbounded)
  for (int a = tid; a < m0c; a += PRE_THREADS) {
    const int at = atoms_g[a];
    sm.atom[a] = at;
    sm.nA[a] = pl.ver_n[(size_t)u * dm.vmax + at];
  }
  if (tid == 0) {
    mbar_init(&sm.bar_mma, 1);
    mbar_init(&sm.bar_v, 1);
    mbar_init(&sm.bar_la, 1);
    fence_mbar_init();
    sm.abort = 0;
  }
  if (dm.fenwick) {
    // fixed policy: the states of row o of the tile are the atoms (tree nodes
    // of [0, T0)), the binary-counter blocks of [T0, T0 + o) (one per set
    // bit of o) and {T0 + o}; the weight pass derives them from o directly
    if (tid == 0) {
      sm.m0 = m0;
      sm.len = min(M, Tw - T0);
      sm.np = 0;
    }
  } else if (warp == 2 && lane == 0) {
    // in-tile pieces and the state partition of each epoch
    const int nev = pl.tile_nev[(size_t)u * dm.tiles + c];
    const int32_t *evo = pl.tile_ev_off + ((size_t)u * dm.tiles + c) * M;
    const int32_t *evm = pl.tile_ev_mrg + ((size_t)u * dm.tiles + c) * M;
    const int len = min(M, Tw - T0);
    sm.m0 = m0;
    sm.len = len;
    const bool cont = !(nev > 0 && evo[0] == 0);
    int np = 0;
    if (cont) sm.pst[np++] = 0;
    for (int i = 0; i < nev; i++) sm.pst[np++] = evo[i];
    for (int p = 0; p < np; p++) sm.pen[p] = p + 1 < np ? sm.pst[p + 1] : len;
    sm.np = np;
    sm.cont = cont ? 1 : 0;
    // unbounded policy: no merges, so every atom and piece ends a state of
    // its own except the last atom when piece 0 continues it (no bitmask)
    if (!dm.unb) {
    uint32_t cur[BW];
    for (int w = 0; w < BW; w++)
      cur[w] = m0 >= 32 * (w + 1) ? ~0u : (m0 > 32 * w ? (1u << (m0 - 32 * w)) - 1u : 0u);
    for (int p = 0; p < np; p++) {
      const int beta = m0 + p;
      if (p == 0 && cont) {
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
    }
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = sm.tmem_base;
  const int np = sm.np, len = sm.len;
  if (tid < M && !dm.fenwick) {  // piece of each row (rows past the tile's end take the last piece)
    int p = 0;
    while (p + 1 < np && sm.pst[p + 1] <= tid) p++;
    sm.pidx[tid] = p;
  }

  mbar_wait(&sm.bar_load, 0, abort);

  // ---- Mu (bf16 means of the atoms) -------------------------------------------
  const int n_mu = (m0c + 15) & ~15;
  for (int e = tid; e < n_mu * 16; e += PRE_THREADS) {
    const int a = e >> 4, ch = e & 15;
    uint4 x = make_uint4(0, 0, 0, 0);
    if (a < m0c) {
      const float4 *zz = reinterpret_cast<const float4 *>(pl.ver_z + ((size_t)u * dm.vmax + sm.atom[a]) * D + ch * 8);
      const float inv = 1.0f / sm.nA[a];
      const float4 z0 = zz[0], z1 = zz[1];
      x.x = pack_bf16(z0.x * inv, z0.y * inv);
      x.y = pack_bf16(z0.z * inv, z0.w * inv);
      x.z = pack_bf16(z1.x * inv, z1.y * inv);
      x.w = pack_bf16(z1.z * inv, z1.w * inv);
    }
    *reinterpret_cast<uint4 *>(mu_buf + sw128_offset(a, ch * 8, 128)) = x;
  }
  fence_proxy_async();
  tc_fence_before();
  __syncthreads();

  const uint32_t q_s = smem_u32(sm.q), kp_s = smem_u32(sm.kp);
  auto kdesc = [](uint32_t base, int k) {  // K-major SW128, 128 rows per half
    return sdesc(base + (k >> 2) * (TILE_BYTES / 2) + (k & 3) * 32, 16, 1024);
  };
  // ---- A = phi(Q) phi(K)^T and LA = phi(Q) Mu^T ------------------------------
  if (warp == 1 && lane == 0) {
    tc_fence_after();
    for (int k = 0; k < 8; k++)
      mma_bf16(tbase + PRE_A, kdesc(q_s, k), kdesc(kp_s, k), idesc_bf16(M, 128, 0, 0), k > 0);
    if (m0 > 0)
      for (int k = 0; k < 8; k++)
        mma_bf16(tbase + PRE_LA, kdesc(q_s, k), kdesc(smem_u32(mu_buf), k),
                 idesc_bf16(M, n_mu, 0, 0), k > 0);
    mma_commit(&sm.bar_mma);
  }
  mbar_wait(&sm.bar_mma, 0, abort);
  tc_fence_after();
  if (tid == 0) {  // phi(K) has been read: the v tile takes its place
    mbar_expect_tx(&sm.bar_v, TILE_BYTES);
    for (int h = 0; h < 2; h++)
      tma_load_3d(sm.kp + h * (TILE_BYTES / 2), &tv, &sm.bar_v, h * 64, ca.w0 + T0, u);
  }

  // ---- unbounded policy: the atoms' logits, 128 at a time ----------------------
  // With no merges every atom is a state of its own, except the last one
  // when piece 0 continues it (the open state), so no segmented sums are
  // needed.  Chunk 0's logits came with A; each further chunk's means replace
  // Mu and its logits LA (all threads take part: shared Mu, one MMA thread).
  // The row warps keep the softmax's running maximum and sum over the atoms
  // that end a state and park each atom's scaled logit in the plan's weight
  // array, rewritten as its weight once the maximum and sum are final.
  float u_mx = -INFINITY, u_l = 0.f, u_lalast = 0.f;
  if (dm.unb) {
    const bool rw = warp >= 4 && warp < 8;
    const int qd = warp & 3;
    const int t = 32 * qd + lane;
    const uint32_t trow = tbase + ((uint32_t)(32 * qd) << 16);
    const bool last_joins = sm.cont && m0 > 0;
    for (int a0 = 0; a0 < m0; a0 += 128) {
      const int na = min(128, m0 - a0);
      if (a0 > 0) {
        const int nmu = (na + 15) & ~15;
        for (int e = tid; e < nmu * 16; e += PRE_THREADS) {
          const int a = e >> 4, ch = e & 15;
          uint4 x = make_uint4(0, 0, 0, 0);
          if (a < na) {
            const int at = atoms_g[a0 + a];
            const float4 *zz = reinterpret_cast<const float4 *>(pl.ver_z + ((size_t)u * dm.vmax + at) * D + ch * 8);
            const float inv = 1.0f / pl.ver_n[(size_t)u * dm.vmax + at];
            const float4 z0 = zz[0], z1 = zz[1];
            x.x = pack_bf16(z0.x * inv, z0.y * inv);
            x.y = pack_bf16(z0.z * inv, z0.w * inv);
            x.z = pack_bf16(z1.x * inv, z1.y * inv);
            x.w = pack_bf16(z1.z * inv, z1.w * inv);
          }
          *reinterpret_cast<uint4 *>(mu_buf + sw128_offset(a, ch * 8, 128)) = x;
        }
        fence_proxy_async();
        tc_fence_before();
        __syncthreads();
        if (warp == 1 && lane == 0) {
          tc_fence_after();
          const uint32_t q_s0 = smem_u32(sm.q);
          for (int k = 0; k < 8; k++)
            mma_bf16(tbase + PRE_LA, sdesc(q_s0 + (k >> 2) * (TILE_BYTES / 2) + (k & 3) * 32, 16, 1024),
                     sdesc(smem_u32(mu_buf) + (k >> 2) * (TILE_BYTES / 2) + (k & 3) * 32, 16, 1024),
                     idesc_bf16(M, nmu, 0, 0), k > 0);
          mma_commit(&sm.bar_la);
        }
        mbar_wait(&sm.bar_la, ((a0 >> 7) - 1) & 1, abort);
        tc_fence_after();
      }
      if (rw) {
#pragma unroll 1
        for (int b = 0; b * 32 < na; b++) {
          uint32_t r[32];
          DLA_TMEM_LD32(trow + PRE_LA + 32 * b, r);
          tmem_wait_ld();
          float x[32];
#pragma unroll
          for (int j = 0; j < 32; j++) {
            const int a = a0 + 32 * b + j;
            const bool joins = last_joins && a == m0 - 1;
            u_lalast = joins ? __uint_as_float(r[j]) : u_lalast;
            x[j] = (a < m0 && !joins) ? __uint_as_float(r[j]) * INV_SQRT_D : -INFINITY;
          }
          const float cmx = max32(x);
          if (cmx > -INFINITY) {
            float e[32];
#pragma unroll
            for (int j = 0; j < 32; j++) e[j] = __expf(x[j] - cmx);
            const float cl = sum32(e);
            const float nm = fmaxf(u_mx, cmx);
            u_l = u_l * __expf(u_mx - nm) + cl * __expf(cmx - nm);
            u_mx = nm;
          }
#pragma unroll
          for (int j = 0; j < 32; j++)
            if (a0 + 32 * b + j < m0) preW[(size_t)(a0 + 32 * b + j) * M + t] = x[j];
        }
      }
      tc_fence_before();
      __syncthreads();
    }
  }

  // ---- softmax weights per row (warps 4..7, row t = TMEM lane) ----------------
  // Pass A walks the row's atoms (TMEM columns, 32 at a time) and pieces in
  // time order: segmented sums of x_beta and n_beta give each state's logit at
  // its last atom / piece (written in place); the softmax max and sum are
  // merged once per chunk.  Pass B walks backwards and gives every atom /
  // piece the weight of the state it belongs to.  Piece values live in
  // registers when there are at most PREG pieces, else in the tile's O_intra
  // slot of the plan (written only at the end).  P replaces A in place.
  if (dm.fenwick && warp >= 4 && warp < 8) {
    // Row o: block sums of A[o][s] over the row's in-tile blocks (s < o lies
    // in the block of size 2^p, p = the highest bit where s and o differ),
    // one softmax over atoms, blocks and {o}, then P[o][s] = w(block) A[o][s].
    const int qd = warp & 3;
    const int t = 32 * qd + lane;
    const uint32_t trow = tbase + ((uint32_t)(32 * qd) << 16);
    float bsum[7];
#pragma unroll
    for (int q = 0; q < 7; q++) bsum[q] = 0.f;
    float aself = 0.f;
#pragma unroll 1
    for (int s0 = 0; s0 < M; s0 += 8) {
      uint32_t ar[8];
      DLA_TMEM_LD8(trow + PRE_A + s0, ar);
      tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 8; j++) {
        const int s = s0 + j;
        const float x = __uint_as_float(ar[j]);
        const int pb = 31 - __clz(s ^ t);
#pragma unroll
        for (int q = 0; q < 7; q++) bsum[q] += (s < t && pb == q) ? x : 0.f;
        aself = s == t ? x : aself;
      }
    }
    float lg[7];
    float mx = aself * INV_SQRT_D;
#pragma unroll
    for (int q = 0; q < 7; q++) {
      lg[q] = bsum[q] * (1.0f / (float)(1 << q)) * INV_SQRT_D;
      if ((t >> q) & 1) mx = fmaxf(mx, lg[q]);
    }
#pragma unroll 1
    for (int a0 = 0; a0 < m0; a0 += 8) {
      uint32_t r[8];
      DLA_TMEM_LD8(trow + PRE_LA + a0, r);
      tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 8; j++)
        if (a0 + j < m0) mx = fmaxf(mx, __uint_as_float(r[j]) * INV_SQRT_D);
    }
    float l = __expf(aself * INV_SQRT_D - mx);
#pragma unroll
    for (int q = 0; q < 7; q++)
      if ((t >> q) & 1) l += __expf(lg[q] - mx);
#pragma unroll 1
    for (int a0 = 0; a0 < m0; a0 += 8) {
      uint32_t r[8];
      DLA_TMEM_LD8(trow + PRE_LA + a0, r);
      tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 8; j++)
        if (a0 + j < m0) l += __expf(__uint_as_float(r[j]) * INV_SQRT_D - mx);
    }
    const float inv_l = 1.0f / l;
#pragma unroll 1
    for (int a0 = 0; a0 < m0; a0 += 8) {
      uint32_t r[8];
      DLA_TMEM_LD8(trow + PRE_LA + a0, r);
      tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 8; j++)
        if (a0 + j < m0) preW[(a0 + j) * M + t] = __expf(__uint_as_float(r[j]) * INV_SQRT_D - mx) * inv_l;
    }
    float wb[7];
#pragma unroll
    for (int q = 0; q < 7; q++) wb[q] = ((t >> q) & 1) ? __expf(lg[q] - mx) * inv_l : 0.f;
    const float wself = __expf(aself * INV_SQRT_D - mx) * inv_l;
#pragma unroll 1
    for (int s0 = 0; s0 < M; s0 += 8) {
      uint32_t ar[8];
      DLA_TMEM_LD8(trow + PRE_A + s0, ar);
      tmem_wait_ld();
      uint32_t pk[4];
#pragma unroll
      for (int j = 0; j < 8; j += 2) {
        float v2[2];
#pragma unroll
        for (int h = 0; h < 2; h++) {
          const int s = s0 + j + h;
          const int pb = 31 - __clz(s ^ t);
          float w = 0.f;
#pragma unroll
          for (int q = 0; q < 7; q++) w = (pb == q) ? wb[q] : w;
          w = s < t ? w : (s == t ? wself : 0.f);
          v2[h] = (s < len) ? w * __uint_as_float(ar[j + h]) : 0.f;
        }
        pk[j >> 1] = pack_bf16(v2[0], v2[1]);
      }
      DLA_TMEM_ST4(trow + p_col(s0), pk);
    }
    tmem_wait_st();
  } else if (warp >= 4 && warp < 8) {
    // One thread per row, blocks of 32 columns / atoms: one TMEM load per
    // block and 32 independent operations per step (a single warp per
    // scheduler cannot hide dependent latencies).  Piece boundaries are the
    // same for every row, so the loops over them are warp-uniform; a block
    // whose atoms are all states of their own (the common case) needs no
    // segmented sums: its logits are LA / sqrt(d).
    constexpr int PREG = 8;
    const int qd = warp & 3;
    const int t = 32 * qd + lane;
    const uint32_t trow = tbase + ((uint32_t)(32 * qd) << 16);
    const int ep = sm.pidx[t];
    const uint32_t *bits = sm.bits + ep * BW;
    const int smax = min(32 * qd + 31, len - 1);  // last column a row of this warp reads
    float pv[PREG];  // piece sums, then logits, then weights
    float *const ovf = reinterpret_cast<float *>(sm.q);  // pieces PREG.. (rows in columns)
#pragma unroll
    for (int k = 0; k < PREG; k++) pv[k] = 0.f;
    auto piece_get = [&](int p) -> float {
      if (p < PREG) {
        float x = 0.f;
#pragma unroll
        for (int k = 0; k < PREG; k++) x = (k == p) ? pv[k] : x;
        return x;
      }
      return ovf[(size_t)p * M + t];
    };
    auto piece_put = [&](int p, float x) {
      if (p < PREG) {
#pragma unroll
        for (int k = 0; k < PREG; k++) pv[k] = (k == p) ? x : pv[k];
      } else {
        ovf[(size_t)p * M + t] = x;
      }
    };
    // piece sums y_p(t) = sum_{s in p, s <= t} A[t][s]; pieces that start
    // past the warp's last row are never read (p > ep for all its rows)
    {
      float y = 0.f;
      int p = 0;
      int nxt = np > 1 ? sm.pst[1] : M + 1;
#pragma unroll 1
      for (int s0 = 0; s0 <= smax; s0 += 32) {
        uint32_t ar[32];
        DLA_TMEM_LD32(trow + PRE_A + s0, ar);
        tmem_wait_ld();
        float x[32];
#pragma unroll
        for (int j = 0; j < 32; j++) x[j] = (s0 + j <= t && s0 + j < len) ? __uint_as_float(ar[j]) : 0.f;
        int lo = s0;
#pragma unroll 1
        while (true) {
          const int hi = min(nxt, s0 + 32);
          float xs[32];
#pragma unroll
          for (int j = 0; j < 32; j++) xs[j] = (s0 + j >= lo && s0 + j < hi) ? x[j] : 0.f;
          y += sum32(xs);
          if (nxt >= s0 + 32) break;
          piece_put(p, y);
          p++;
          y = 0.f;
          lo = nxt;
          nxt = p + 1 < np ? sm.pst[p + 1] : M + 1;
        }
      }
      piece_put(p, y);
    }
    // pass A: each state's logit at its last atom / piece, online softmax max
    // and sum; atom columns keep exp(logit - block max) (0 for atoms that do
    // not end a state), pieces keep their logits.  Under the unbounded policy
    // the atoms were done chunk by chunk above; the last atom joins piece 0
    // when the tile continues the open state.
    float mx = -INFINITY, l = 0.f, sacc = 0.f, nacc = 0.f;
    float bmx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};  // block maxima
    const bool unb = dm.unb != 0;
    if (unb) {
      mx = u_mx;
      l = u_l;
      if (sm.cont && m0 > 0) {
        const float nn = pl.ver_n[(size_t)u * dm.vmax + atoms_g[m0 - 1]];
        sacc = nn * u_lalast;
        nacc = nn;
      }
    }
#pragma unroll 1
    for (int b = 0; !unb && b * 32 < m0; b++) {
      const int a0 = b * 32;
      uint32_t r[32];
      DLA_TMEM_LD32(trow + PRE_LA + a0, r);
      const int nval = min(32, m0 - a0);
      const uint32_t vmask = nval == 32 ? ~0u : (1u << nval) - 1u;
      const uint32_t wb = bits[b] & vmask;
      const bool fast = wb == vmask && (b == 0 || (bits[b - 1] >> 31));
      tmem_wait_ld();
      float a[32];
      if (__all_sync(0xffffffffu, fast)) {
#pragma unroll
        for (int j = 0; j < 32; j++) a[j] = j < nval ? __uint_as_float(r[j]) * INV_SQRT_D : -INFINITY;
      } else {
        float s = sacc, n = nacc;
#pragma unroll
        for (int j = 0; j < 32; j++) {
          const bool valid = j < nval, end = (wb >> j) & 1u;
          const float nn = sm.nA[a0 + j];
          s = valid ? fmaf(nn, __uint_as_float(r[j]), s) : s;
          n = valid ? n + nn : n;
          a[j] = end ? __fdividef(s, n) * INV_SQRT_D : -INFINITY;
          s = end ? 0.f : s;
          n = end ? 0.f : n;
        }
        sacc = s;
        nacc = n;
      }
      const float cmx = max32(a);
      if (cmx > -INFINITY) {
#pragma unroll
        for (int j = 0; j < 32; j++) a[j] = __expf(a[j] - cmx);
        const float cl = sum32(a);
        const float nm = fmaxf(mx, cmx);
        l = l * __expf(mx - nm) + cl * __expf(cmx - nm);
        mx = nm;
      } else {
#pragma unroll
        for (int j = 0; j < 32; j++) a[j] = 0.f;
      }
#pragma unroll
      for (int k = 0; k < 4; k++) bmx[k] = (k == b) ? cmx : bmx[k];
#pragma unroll
      for (int j = 0; j < 32; j++) r[j] = __float_as_uint(a[j]);
      DLA_TMEM_ST32(trow + PRE_LA + a0, r);
      tmem_wait_st();
    }
#pragma unroll 1
    for (int p = 0; p < np; p++) {
      float y = piece_get(p);
      if (p <= ep) {
        const float nn = p < ep ? (float)(sm.pen[p] - sm.pst[p]) : (float)(t - sm.pst[p] + 1);
        sacc += y;
        nacc += nn;
        if (unb || bit_of(bits, m0 + p)) {
          const float a = __fdividef(sacc, nacc) * INV_SQRT_D;
          y = a;
          const float nm = fmaxf(mx, a);
          l = l * __expf(mx - nm) + __expf(a - nm);
          mx = nm;
          sacc = 0.f;
          nacc = 0.f;
        }
      }
      piece_put(p, y);
    }
    // pass B (reverse): every atom / piece gets the weight of its state
    const float inv_l = 1.0f / l;
    float cur = 0.f;
#pragma unroll 1
    for (int p = np - 1; p >= 0; p--) {
      const float a = piece_get(p);
      float w = 0.f;
      if (p <= ep) {
        if (unb || bit_of(bits, m0 + p)) cur = __expf(a - mx) * inv_l;
        w = cur;
      }
      piece_put(p, w);
    }
    if (unb) {
      // every atom's weight from its parked logit; the last one shares
      // piece 0's state when it continues into the tile
      const float w0 = piece_get(0);
      const bool last_joins = sm.cont && m0 > 0;
#pragma unroll 4
      for (int a = 0; a < m0; a++) {
        float *pw = preW + (size_t)a * M + t;
        *pw = (last_joins && a == m0 - 1) ? w0 : __expf(*pw - mx) * inv_l;
      }
    }
#pragma unroll 1
    for (int b = (m0 - 1) >> 5; !unb && m0 > 0 && b >= 0; b--) {
      const int a0 = b * 32;
      uint32_t r[32];
      DLA_TMEM_LD32(trow + PRE_LA + a0, r);
      const int nval = min(32, m0 - a0);
      const uint32_t vmask = nval == 32 ? ~0u : (1u << nval) - 1u;
      const uint32_t wb = bits[b] & vmask;
      const bool fast = wb == vmask && (b == 0 || (bits[b - 1] >> 31));
      float cb = bmx[0];
#pragma unroll
      for (int k = 1; k < 4; k++) cb = (k == b) ? bmx[k] : cb;
      const float f = cb > -INFINITY ? __expf(cb - mx) * inv_l : 0.f;
      tmem_wait_ld();
      if (__all_sync(0xffffffffu, fast)) {
        // the atom before the block ends a state, so no weight carries over
#pragma unroll
        for (int j = 0; j < 32; j++) r[j] = __float_as_uint(__uint_as_float(r[j]) * f);
      } else {
#pragma unroll
        for (int j = 31; j >= 0; j--) {
          if (j < nval) {
            if ((wb >> j) & 1u) cur = __uint_as_float(r[j]) * f;
            r[j] = __float_as_uint(cur);
          }
        }
      }
#pragma unroll
      for (int j = 0; j < 32; j++)
        if (j < nval) preW[(a0 + j) * M + t] = __uint_as_float(r[j]);
    }
    // P[t][s] = W_{piece(s)}(t) A[t][s] for s <= t, as the bf16 A operand of
    // P V; columns past the warp's last row are zero
    {
      int p = 0;
      float w = piece_get(0);
      int nxt = np > 1 ? sm.pst[1] : M + 1;
#pragma unroll 1
      for (int s0 = 0; s0 < M; s0 += 32) {
        uint32_t pk[16];
#pragma unroll
        for (int j = 0; j < 16; j++) pk[j] = 0u;
        if (s0 <= smax) {
          uint32_t ar[32];
          DLA_TMEM_LD32(trow + PRE_A + s0, ar);
          tmem_wait_ld();
          float v[32];
#pragma unroll
          for (int j = 0; j < 32; j++) v[j] = 0.f;
          int lo = s0;
#pragma unroll 1
          while (true) {
            const int hi = min(nxt, s0 + 32);
#pragma unroll
            for (int j = 0; j < 32; j++)
              v[j] = (s0 + j >= lo && s0 + j < hi) ? w * __uint_as_float(ar[j]) : v[j];
            if (nxt >= s0 + 32) break;
            p++;
            w = piece_get(p);
            lo = nxt;
            nxt = p + 1 < np ? sm.pst[p + 1] : M + 1;
          }
#pragma unroll
          for (int j = 0; j < 16; j++) {
            const int s = s0 + 2 * j;
            pk[j] = pack_bf16((s <= t && s < len) ? v[2 * j] : 0.f, (s + 1 <= t && s + 1 < len) ? v[2 * j + 1] : 0.f);
          }
        }
        DLA_TMEM_ST16(trow + p_col(s0), pk);
      }
      tmem_wait_st();
    }
  }
  fence_proxy_async();
  tc_fence_before();
  __syncthreads();

  // ---- O_intra = P V, stored for the atom loop -------------------------------
  if (warp == 1 && lane == 0) {
    const bool ok = mbar_wait(&sm.bar_v, 0, abort);
    tc_fence_after();
    if (ok)
      for (int k = 0; k < 8; k++)
        mma_bf16_ta(tbase + PRE_LA, tbase + pa_col(k), sdesc(kp_s + k * 2048, TILE_BYTES / 2, 1024),
                    idesc_bf16(M, 128, 0, 1), k > 0);
    mma_commit(&sm.bar_mma);
  }
  mbar_wait(&sm.bar_mma, 1, abort);
  tc_fence_after();
  {
    const int qd = warp & 3, hc = warp >> 2;
    const int t = 32 * qd + lane;
    const uint32_t trow = tbase + ((uint32_t)(32 * qd) << 16);
    uint4 *dst = reinterpret_cast<uint4 *>(pl.pre_o) + g * (M * D / 8);
#pragma unroll
    for (int half = 0; half < 2; half++) {
      uint32_t pr[32];
      DLA_TMEM_LD32(trow + PRE_LA + hc * 64 + 32 * half, pr);
      tmem_wait_ld();
#pragma unroll
      for (int i = 0; i < 4; i++)
        dst[pre_o_chunk(t, hc, 4 * half + i)] =
            make_uint4(pack_bf16(__uint_as_float(pr[8 * i]), __uint_as_float(pr[8 * i + 1])),
                       pack_bf16(__uint_as_float(pr[8 * i + 2]), __uint_as_float(pr[8 * i + 3])),
                       pack_bf16(__uint_as_float(pr[8 * i + 4]), __uint_as_float(pr[8 * i + 5])),
                       pack_bf16(__uint_as_float(pr[8 * i + 6]), __uint_as_float(pr[8 * i + 7])));
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, PRE_COLS);
  }
  if (tid == 0 && sm.abort) set_status(ca.dev_status, DLA_ERR_TIMEOUT);
}

// The atom loop: each CTA walks a run of consecutive tiles of one head.
// Tensor memory is allocated and the barriers set up once per run; stage,
// product-buffer and weight-chunk phases follow cumulative counters over the
// run's tiles, so each role runs ahead into the next tile as far as its
// barriers let it.  phi(Q) has a landing buffer of its own and two
// tensor-memory regions (by tile parity): the next tile's phi(Q) loads while
// this tile's MMAs run, and the epilogue moves it into tensor memory as soon
// as it starts that tile.  The prologue's weights stream through a ring of
// WCH-atom chunks; its intra-tile output is the accumulator's start.  The
// producer also prefetches the run's next tile (weights, intra-tile output,
// first versions) into L2.
__global__ void __launch_bounds__(THREADS, 1)
    k_readout_tc(const __grid_constant__ CUtensorMap tq, Dims dm, Plan pl, CallArgs ca, int run) {
  extern __shared__ uint8_t raw[];
  Smem &sm = *reinterpret_cast<Smem *>((reinterpret_cast<uintptr_t>(raw) + 1023) &
                                       ~static_cast<uintptr_t>(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  volatile int *abort = &sm.abort;
  // this CTA's run: tiles [c0, c0 + run) of head u (flat index gi = u tiles + c)
  const int runs = (dm.tiles + run - 1) / run;
  const int u = blockIdx.x / runs, c0 = (blockIdx.x % runs) * run;
  const int G = u * dm.tiles + min(dm.tiles, c0 + run);  // one past the run
  const int Tw = tw_of(ca, u);
  // the run's next tile from gi on; a tile at or past the stream's length has
  // no rows, nor has any later one
  auto next_tile = [&](int gi) -> int {
    return gi < G && (gi - u * dm.tiles) * M < Tw ? gi : G;
  };

  const int first = next_tile(u * dm.tiles + c0);
  if (first >= G) return;  // the whole run lies past the stream's length

  // ---- setup (once): TMEM, barriers, the first tile's phi(Q) ----------------
  if (warp == 1) tmem_alloc(&sm.tmem_base, 512);
  if (tid == 0) {
    mbar_init(&sm.bar_load, 1);
    mbar_init(&sm.bar_qa, 8);
    mbar_init(&sm.bar_qs, 2);
    for (int i = 0; i < NSV; i++) {
      mbar_init(&sm.full[i], 1);
      mbar_init(&sm.empty[i], 1);
    }
    for (int i = 0; i < NPB; i++) {
      mbar_init(&sm.tfull[i], 1);
      mbar_init(&sm.tempty[i], 8);
    }
    for (int i = 0; i < NWC; i++) {
      mbar_init(&sm.wfull[i], 1);
      mbar_init(&sm.wempty[i], 8);
    }
    fence_mbar_init();
    sm.abort = 0;
    mbar_expect_tx(&sm.bar_load, TILE_BYTES);
    for (int h = 0; h < 2; h++)
      tma_load_3d(sm.q + h * (TILE_BYTES / 2), &tq, &sm.bar_load, h * 64, (first - u * dm.tiles) * M, u);
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = sm.tmem_base;
  auto kdesc = [](uint32_t base, int k) {  // K-major SW128, 128 rows per half
    return sdesc(base + (k >> 2) * (TILE_BYTES / 2) + (k & 3) * 32, 16, 1024);
  };

  if (warp == 0 && lane == 0) {
    // ---- producer: versions (L2 prefetch PF atoms ahead), weight chunks,
    // and the next tile's phi(Q) once this tile's is in tensor memory -------
    constexpr int PF = 6;
    // a tile's weights, intra-tile output and first versions, into L2 a tile
    // ahead of their loads
    auto prefetch_tile = [&](int gp) {
      if (gp >= G) return;
      const int mp = pl.tile_m0[gp];
      if (mp > 0) bulk_prefetch_l2(pl.pre_w + (size_t)gp * dm.amax * M, (uint32_t)mp * M * 4);
      bulk_prefetch_l2(static_cast<const uint8_t *>(pl.pre_o) + (size_t)gp * M * D * 2, M * D * 2);
      const int32_t *ap = pl.tile_atoms + (size_t)gp * dm.amax;
      const uint8_t *vp = static_cast<const uint8_t *>(pl.ver_S) +
                          (size_t)u * dm.vmax * VER_BYTES;
      for (int a = 0; a < mp && a < PF; a++) bulk_prefetch_l2(vp + (size_t)ap[a] * VER_BYTES, VER_BYTES);
    };
    uint32_t A0 = 0, W0 = 0;
    int it = 0;
    for (int gi = first; gi < G; gi = next_tile(gi + 1), it++) {
      const int m0 = pl.tile_m0[gi];
      const int32_t *atoms = pl.tile_atoms + (size_t)gi * dm.amax;
      const uint8_t *verS = static_cast<const uint8_t *>(pl.ver_S) + (size_t)u * dm.vmax * VER_BYTES;
      const float *wsrc = pl.pre_w + (size_t)gi * dm.amax * M;
      if (it == 0) prefetch_tile(gi);
      prefetch_tile(next_tile(gi + 1));
      bool qdone = false;
      auto next_q = [&]() {  // the next tile's phi(Q), once this one's is moved
        qdone = true;
        const int gn = next_tile(gi + 1);
        if (gn >= G) return;
        // the landing buffer is free once this tile's phi(Q) is in tensor
        // memory, and both issuers must have seen that before the barrier
        // can complete again (an issuer with no atoms in a tile still takes
        // its phase, so its parity waits never fall two phases behind)
        if (!mbar_wait(&sm.bar_qa, it & 1, abort) || !mbar_wait(&sm.bar_qs, it & 1, abort)) return;
        mbar_expect_tx(&sm.bar_load, TILE_BYTES);
        for (int h = 0; h < 2; h++)
          tma_load_3d(sm.q + h * (TILE_BYTES / 2), &tq, &sm.bar_load, h * 64, (gn - u * dm.tiles) * M, u);
      };
      for (int a = 0; a < m0; a++) {
        if (a % WCH == 0) {
          const uint32_t k = W0 + a / WCH;
          const int w = (int)(k % NWC);
          if (k >= NWC && !mbar_wait(&sm.wempty[w], (int)((k / NWC) - 1) & 1, abort)) break;
          const uint32_t nb = (uint32_t)min(WCH, m0 - a) * M * 4;
          mbar_expect_tx(&sm.wfull[w], nb);
          bulk_load(sm.w[w], wsrc + (size_t)a * M, nb, &sm.wfull[w]);
        }
        if (a + PF < m0) bulk_prefetch_l2(verS + (size_t)atoms[a + PF] * VER_BYTES, VER_BYTES);
        const uint32_t x = A0 + a;
        const int s = (int)(x % NSV);
        if (x >= NSV && !mbar_wait(&sm.empty[s], (int)((x / NSV) - 1) & 1, abort)) break;
        mbar_expect_tx(&sm.full[s], VER_BYTES);
        bulk_load(sm.st[s], verS + (size_t)atoms[a] * VER_BYTES, VER_BYTES, &sm.full[s]);
        if (a == NSV - 1) next_q();
      }
      if (!qdone) next_q();
      A0 += m0;
      W0 += (m0 + WCH - 1) / WCH;
    }
  } else if ((warp == 1 || warp == 2) && lane == 0) {
    // ---- two MMA issuers: even / odd atoms of the CTA's running count ------
    // (an issuing thread is held for about the duration of its MMAs, so with
    // one issuer every barrier wait left the tensor pipe idle).  Atom x goes
    // to product buffer x % 3: three buffers cover a buffer's round trip
    // (MMAs, commit, epilogue drain, release) at the MMA rate.
    tc_fence_after();
    const int par_i = warp - 1;
    uint32_t A0 = 0;
    int it = 0;
    for (int gi = first; gi < G; gi = next_tile(gi + 1), it++) {
      const int m0 = pl.tile_m0[gi];
      // every tile's phi(Q) phase is taken, atoms or not, and acknowledged
      const bool ok_qa = mbar_wait(&sm.bar_qa, it & 1, abort);
      mbar_arrive(&sm.bar_qs);
      {
        int a = (int)((par_i - (A0 & 1) + 2) & 1);  // first atom of this issuer's parity
        for (; a < m0; a += 2) {
          const uint32_t x = A0 + a;
          const int s = (int)(x % NSV), b = (int)(x % NPB);
          bool ok = mbar_wait(&sm.full[s], (int)(x / NSV) & 1, abort) && ok_qa;
          if (x >= NPB) ok = mbar_wait(&sm.tempty[b], (int)((x / NPB) - 1) & 1, abort) && ok;
          tc_fence_after();
          if (ok) {
            const uint32_t st_s = smem_u32(sm.st[s]);
            for (int k = 0; k < 8; k++)
              mma_bf16_ta(tbase + pbuf_col(b), tbase + qa_col(k, it & 1), kdesc(st_s, k),
                          idesc_bf16(M, 128, 0, 0), k > 0);
          }
          mma_commit(&sm.empty[s]);
          mma_commit(&sm.tfull[b]);
        }
      }
      A0 += m0;
    }
  } else if (warp >= 4) {
    // ---- 8 epilogue warps: row t = 32 qd + lane, columns [64 hc, 64 hc + 64)
    const int qd = warp & 3, hc = (warp - 4) >> 2;
    const int t = 32 * qd + lane;
    const uint32_t trow = tbase + ((uint32_t)(32 * qd) << 16);
    uint32_t A0 = 0, W0 = 0;
    int it = 0;
    for (int gi = first; gi < G; gi = next_tile(gi + 1), it++) {
      const int c = gi - u * dm.tiles;
      const int T0 = c * M;
      const int len = min(M, tw_of(ca, u) - T0);
      const int m0 = pl.tile_m0[gi];
      // the intra-tile output, the accumulator's start (in flight during the
      // phi(Q) move)
      const uint4 *src = reinterpret_cast<const uint4 *>(pl.pre_o) + (size_t)gi * (M * D / 8);
      uint4 po[8];
#pragma unroll
      for (int i = 0; i < 8; i++) po[i] = src[pre_o_chunk(t, hc, i)];
      // this tile's phi(Q) rows into its tensor-memory region (the region's
      // last reader, tile it - 2, is done: this warp drained all its products)
      mbar_wait(&sm.bar_load, it & 1, abort);
      {
        uint32_t qw[32];
#pragma unroll
        for (int i = 0; i < 8; i++) {
          const uint4 x = *reinterpret_cast<const uint4 *>(sm.q + sw128_offset(t, 64 * hc + 8 * i, M));
          qw[4 * i] = x.x;
          qw[4 * i + 1] = x.y;
          qw[4 * i + 2] = x.z;
          qw[4 * i + 3] = x.w;
        }
        DLA_TMEM_ST32(trow + COL_AI + 32 * (it & 1) + 64 * hc, qw);
        tmem_wait_st();
      }
      // the landing buffer is read (the next tile's phi(Q) may overwrite it)
      fence_proxy_async();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.bar_qa);
      float acc[64];
#pragma unroll
      for (int i = 0; i < 8; i++) {
        acc[8 * i] = bf16_lo(po[i].x);
        acc[8 * i + 1] = bf16_hi(po[i].x);
        acc[8 * i + 2] = bf16_lo(po[i].y);
        acc[8 * i + 3] = bf16_hi(po[i].y);
        acc[8 * i + 4] = bf16_lo(po[i].z);
        acc[8 * i + 5] = bf16_hi(po[i].z);
        acc[8 * i + 6] = bf16_lo(po[i].w);
        acc[8 * i + 7] = bf16_hi(po[i].w);
      }
#pragma unroll 1
      for (int a = 0; a < m0; a++) {
        const uint32_t k = W0 + a / WCH;
        const int w = (int)(k % NWC);
        if (a % WCH == 0) mbar_wait(&sm.wfull[w], (int)(k / NWC) & 1, abort);
        const float wt = sm.w[w][(a % WCH) * M + t];
        const uint32_t x = A0 + a;
        const int b = (int)(x % NPB);
        mbar_wait(&sm.tfull[b], (int)(x / NPB) & 1, abort);
        tc_fence_after();
        uint32_t pr[32];
        DLA_TMEM_LD32(trow + pbuf_col(b) + hc * 64, pr);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; i++) acc[i] = fmaf(wt, __uint_as_float(pr[i]), acc[i]);
        DLA_TMEM_LD32(trow + pbuf_col(b) + hc * 64 + 32, pr);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; i++) acc[32 + i] = fmaf(wt, __uint_as_float(pr[i]), acc[32 + i]);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&sm.tempty[b]);
          if (a % WCH == WCH - 1 || a == m0 - 1) mbar_arrive(&sm.wempty[w]);
        }
      }
      // the tile's rows
      if (t < len) {
        uint4 *dst = reinterpret_cast<uint4 *>(static_cast<uint16_t *>(ca.o) +
                                               ((size_t)u * dm.T + ca.w0 + T0 + t) * D + hc * 64);
#pragma unroll
        for (int i = 0; i < 8; i++)
          dst[i] = make_uint4(pack_bf16(acc[8 * i], acc[8 * i + 1]), pack_bf16(acc[8 * i + 2], acc[8 * i + 3]),
                              pack_bf16(acc[8 * i + 4], acc[8 * i + 5]),
                              pack_bf16(acc[8 * i + 6], acc[8 * i + 7]));
      }
      A0 += m0;
      W0 += (m0 + WCH - 1) / WCH;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
  if (tid == 0 && sm.abort) set_status(ca.dev_status, DLA_ERR_TIMEOUT);
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

}  // namespace

bool make_bf16_map_rows(CUtensorMap *m, const void *base, int rows, int stride_rows, int heads);

// 3D tensor map {d = 128, T, heads} of a bf16 [heads][T][128] tensor, boxes of
// 64 x 128 x 1 with the 128-byte swizzle (out-of-range rows read as zero).
bool make_bf16_map(CUtensorMap *m, const void *base, int T, int heads) {
  return make_bf16_map_rows(m, base, T, T, heads);
}
// The same over the first `rows` of every head's `stride_rows` rows.
bool make_bf16_map_rows(CUtensorMap *m, const void *base, int rows, int stride_rows, int heads) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)rows, (cuuint64_t)heads};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)stride_rows * D * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)M, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

namespace {
constexpr int kTileRows = M;
}
int tc_tile_rows() { return kTileRows; }

cudaError_t launch_phi_tc(const Dims &dm, const Plan &pl, const CallArgs &ca, cudaStream_t s) {
  if (dm.D != D || ca.in_dtype != DLA_BF16 || !pl.phi_q) return cudaErrorInvalidValue;
  // 32 KB of (unused) shared memory keeps its CTAs off the SMs that hold
  // the engine, which reserves most of their shared memory
  k_phi_tc<<<148 * 8, 256, 32 * 1024, s>>>(dm, pl, ca);
  return cudaGetLastError();
}

cudaError_t launch_readout_pre_tc(const Dims &dm, const Plan &pl, const CallArgs &ca,
                                  cudaStream_t s) {
  if (dm.M != M || dm.D != D || (dm.C > 128 && !dm.unb) || ca.in_dtype != DLA_BF16 || !pl.phi_q)
    return cudaErrorInvalidValue;
  CUtensorMap tq, tv;
  if (!make_bf16_map_rows(&tq, pl.phi_q, ca.Tw, dm.W, dm.heads) ||
      !make_bf16_map(&tv, ca.v, dm.T, dm.heads))
    return cudaErrorInvalidValue;
  const size_t sb = sizeof(PreSmem) + 1024;
  cudaError_t e = cudaFuncSetAttribute(k_readout_pre, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)sb);
  if (e != cudaSuccess) return e;
  dim3 g(dm.tiles, dm.heads);
  k_readout_pre<<<g, PRE_THREADS, sb, s>>>(tq, tv, dm, pl, ca);
  return cudaGetLastError();
}

cudaError_t launch_readout_tc(const Dims &dm, const Plan &pl, const CallArgs &ca, cudaStream_t s) {
  if (dm.M != M || dm.D != D || (dm.C > 128 && !dm.unb) || ca.in_dtype != DLA_BF16 || !pl.phi_q)
    return cudaErrorInvalidValue;
  CUtensorMap tq;
  if (!make_bf16_map_rows(&tq, pl.phi_q, ca.Tw, dm.W, dm.heads)) return cudaErrorInvalidValue;
  const size_t sb = sizeof(Smem) + 1024;
  cudaError_t e = cudaFuncSetAttribute(k_readout_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)sb);
  if (e != cudaSuccess) return e;
  // tiles per CTA: the CTAs in flight then cover run x (SM count) tiles, and
  // the versions those tiles read must stay in L2.  A dynamic-policy head
  // holds thousands of versions and one tile per CTA keeps the working set
  // to about two heads' tiles in flight (longer runs measured slower: 0.67
  // of the tensor peak at 1 tile per CTA, 0.63 at 4, 0.57 at 8 on the
  // T = 8192 prefill); the fixed policy's few versions per head leave room
  // for runs of 4, which save the per-CTA setup (0.21 -> 0.24)
  const int run = dm.fenwick ? 4 : 1;
  const int runs = (dm.tiles + run - 1) / run;
  k_readout_tc<<<dm.heads * runs, THREADS, sb, s>>>(tq, dm, pl, ca, run);
  return cudaGetLastError();
}

}  // namespace dla
