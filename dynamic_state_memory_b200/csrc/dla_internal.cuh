// dla_internal.cuh -- data structures shared by the libdla kernels.
//
// A prefill call is processed in windows of W tokens.  For each window the
// decision kernels (score, segment scan, segment sums, capacity-merge engine)
// turn the keys into a *plan*:
//   - an op list per head that the materializer executes in time order on the
//     fp32 slot states of the cache (ZERO / ADD tokens / MERGE / SHADOW);
//   - per readout tile (M tokens): the states present just before the tile
//     ("atoms", as frozen versions written by SHADOW ops) and the in-tile
//     boundaries with their merges.
// The readout kernels then treat every tile independently.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/dla.h"

namespace dla {

// Ops of the state materializer.  The open state is kept in registers: ZERO
// or LOAD makes `slot` the register-resident open state, ADD / ADDP
// accumulate tokens into it, STORE writes it back to its slot; MERGE works on
// memory, MERGEO adds the open registers into a sealed slot (the open state
// is the merge's right member and disappears), SHADOW freezes a version (of
// the open registers, or of a sealed slot read from memory).  STORE, MERGE
// and MERGEO carry in .w the version id + 1 of the result (0: none), so a
// sealed state's version is written from registers without a re-read.
enum OpCode : int32_t {
  OP_ZERO = 0,    // (ZERO, slot)
  OP_ADD = 1,     // (ADD, slot, first window token, count)
  OP_MERGE = 2,   // (MERGE, dst, src, version + 1)
  OP_SHADOW = 3,  // (SHADOW, slot, version)
  OP_LOAD = 4,    // (LOAD, slot)
  OP_STORE = 5,   // (STORE, slot, 0, version + 1)
  OP_ADDP = 6,    // (ADDP, slot, piece id, count): add the tensor-core builder's piece
  OP_MERGEO = 7   // (MERGEO, dst, 0, version + 1)
};

// Pieces shorter than this stay SIMT adds in the materializer.
constexpr int PIECE_MIN = 16;
// Piece ids are tile-based: run k (in token order) of the pieces of tile c
// is piece c * PIECES_PER_TILE + k, so the builder needs only the boundary
// flags and runs concurrently with the capacity-merge engine.
constexpr int PIECES_PER_TILE = 128 / PIECE_MIN;

// pair_loss[C - 1] of a stream belongs to no pair (C states have C - 1
// adjacent pairs).  The information policy writes CACHE_INFO_MARK there (its
// pair entries are densities, not Ward losses) and the unbounded policy
// CACHE_UNBOUNDED_MARK (it keeps no pair losses); the capacity-bounded
// cosine / Ward entry points refuse a cache with a negative entry
// (DLA_ERR_UNSUPPORTED) until dla_cache_init resets it.
constexpr double CACHE_INFO_MARK = -1.0;
constexpr double CACHE_UNBOUNDED_MARK = -2.0;

// Merge code of an in-tile boundary event: -1 none, >= 0 merge of the sealed
// pair at that time-order position, <= -2 merge the two newest sealed states
// (-code - 1) times (binary-counter carries of the fixed policy).
constexpr int32_t EV_NO_MERGE = -1;

struct Dims {
  int32_t heads;   // B * H streams in the call
  int32_t T;       // tokens in the call
  int32_t W;       // window length (multiple of M)
  int32_t M;       // readout tile rows
  int32_t tiles;   // W / M
  int32_t D;       // d_k == d_v
  int32_t C;       // cache capacity (slots)
  int32_t amax;    // max atoms per tile
  int32_t vmax;    // max versions per head per window
  int32_t opsmax;  // max ops per head per window
  int32_t vbytes;  // bytes of one version's S
  int32_t pmax;    // max tensor-core pieces per head per window (0 = none)
  int32_t fenwick; // 1: fixed Fenwick policy (every token a piece; closed-form epochs)
  int32_t info;    // 1: information policy (state score, density merges)
  int32_t unb;     // 1: unbounded policy (no capacity merges; C = storage slots)
};

// Per-window plan, every array strided by head.
struct Plan {
  double *r;           // [heads][W] scores
  uint8_t *b;          // [heads][W] boundary flags
  int32_t *seg_start;  // [heads][W + 1] window-local first token of each piece
  int32_t *nseg;       // [heads]
  double *z_end;       // [heads][W][D] phi(k) sum of each piece's state at its end
  double *z_tile;      // [heads][tiles][D] open state's phi(k) sum before each tile
  double *z_part;      // [heads][W][D] phi(k) sum of each in-tile run, at its first token
  int4 *ops;           // [heads][opsmax]
  int32_t *nops;       // [heads]
  int32_t *tile_m0;    // [heads][tiles]
  int32_t *tile_atoms; // [heads][tiles][amax] version ids
  int32_t *tile_nev;   // [heads][tiles]
  int32_t *tile_ev_off;// [heads][tiles][M] boundary offset inside the tile
  int32_t *tile_ev_mrg;// [heads][tiles][M] merge code (see EV_NO_MERGE)
  float *ver_z;        // [heads][vmax][D] sum of phi(k) of each version (mean = z / n)
  float *ver_n;        // [heads][vmax] token count of each version
  void *ver_S;         // [heads][vmax] versions (fp32 [D][D] or bf16 tiled)
  int32_t *slot_ver;   // [heads][C] engine scratch
  double *phi_tab;     // phi in fp64 of negative bf16 inputs of moderate magnitude
  float *pieces;       // [heads][pmax][D][D] fp32 piece states
  // tensor-core readout: per-tile outputs of the prologue kernel (null on
  // the SIMT path)
  void *phi_q;         // [heads][W][D] bf16 phi(q) of the window's rows
  void *phi_k;         // [heads][tiles][2][128][64] bf16 phi(k) tiles, as in shared memory
  float *pre_w;        // [heads][tiles][amax][M] atom weights
  void *pre_o;         // [heads][tiles][M * D] intra-tile outputs (bf16)
  // information policy: score sum of each window piece's state at the
  // piece's end (the piece's own tokens plus, for a continued open state,
  // its earlier ones)
  double *seg_info;    // [heads][W]
};

struct CallArgs {
  const void *q, *k, *v;
  void *o;
  int32_t in_dtype;
  int32_t w0;         // first token of the window inside the call
  int32_t Tw;         // tokens in this window (of the longest stream when ragged)
  const int32_t *lens;  // ragged call: tokens of each sequence [B] (null: all T)
  int32_t H;          // heads per sequence (stream u is sequence u / H)
  float tau;
  dla_cache cache;
  dla_trace trace;    // boundary == NULL when no trace
  int32_t *dev_status;
  // information policy, carried across the call's windows (null otherwise)
  double *info_S;     // [heads][D * D] fp64 open state, element j of thread i at j * 2D + i
  double *info_aux;   // [heads][4]: |S|^2, the open state's score sum, has-open flag
  double *info_slot;  // [heads][C] score sum of each cache slot's state
};

// Tokens of stream u in this window: the window's length, cut at the
// stream's own sequence length in a ragged call (lens[b], clamped to [0, T]).
__device__ __forceinline__ int tw_of(const CallArgs &ca, int u) {
  if (!ca.lens) return ca.Tw;
  const int L = ca.lens[u / ca.H] - ca.w0;
  return L <= 0 ? 0 : (L < ca.Tw ? L : ca.Tw);
}

__device__ __forceinline__ void set_status(int32_t *st, int32_t code) {
  if (st) atomicCAS(st, 0, code);
}

__device__ __forceinline__ float load_in(const void *p, int32_t dtype, size_t i) {
  if (dtype == DLA_F32) return static_cast<const float *>(p)[i];
  uint32_t b = static_cast<uint32_t>(static_cast<const uint16_t *>(p)[i]) << 16;
  return __uint_as_float(b);
}

__device__ __forceinline__ void store_out(void *p, int32_t dtype, size_t i, float x) {
  if (dtype == DLA_F32) {
    static_cast<float *>(p)[i] = x;
  } else {
    // round to nearest even
    uint32_t u = __float_as_uint(x);
    u += 0x7FFFu + ((u >> 16) & 1u);
    static_cast<uint16_t *>(p)[i] = static_cast<uint16_t>(u >> 16);
  }
}

// phi = elu + 1 in fp64 (decision summaries) and fp32 (states, readout).
__device__ __forceinline__ double phi64(double x) { return x > 0.0 ? x + 1.0 : exp(x); }
__device__ __forceinline__ float phi32(float x) { return x > 0.0f ? x + 1.0f : expf(x); }
// phi for a value that is rounded to bf16 right away (tensor-core operands):
// the fast exponential's error is far below bf16's half-ulp.
__device__ __forceinline__ float phi_bf16op(float x) { return x > 0.0f ? x + 1.0f : __expf(x); }

// Host launchers (one per kernel file).
cudaError_t launch_score(const Dims &dm, const Plan &pl, const CallArgs &ca, int policy,
                         cudaStream_t s);
cudaError_t launch_segscan(const Dims &dm, const Plan &pl, const CallArgs &ca, cudaStream_t s);
cudaError_t launch_segsum(const Dims &dm, const Plan &pl, const CallArgs &ca, cudaStream_t s);
cudaError_t launch_info_score(const Dims &dm, const Plan &pl, const CallArgs &ca, cudaStream_t s);
cudaError_t launch_engine(const Dims &dm, const Plan &pl, const CallArgs &ca, cudaStream_t s);
cudaError_t launch_materialize(const Dims &dm, const Plan &pl, const CallArgs &ca,
                               cudaStream_t s, bool bf16_versions);
cudaError_t launch_phi_tc(const Dims &dm, const Plan &pl, const CallArgs &ca, cudaStream_t s);
cudaError_t launch_readout_pre_tc(const Dims &dm, const Plan &pl, const CallArgs &ca,
                                  cudaStream_t s);
cudaError_t launch_readout_tc(const Dims &dm, const Plan &pl, const CallArgs &ca, cudaStream_t s);
cudaError_t launch_build_tc(const Dims &dm, const Plan &pl, const CallArgs &ca, cudaStream_t s);
cudaError_t launch_fen_leaves_tc(const Dims &dm, const Plan &pl, const CallArgs &ca, float *treeS,
                                 float *treeZ, int nodes, int ntiles, cudaStream_t s);
void fen_tree_shape(int T, int M, int *nodes, int *levels);
// Fixed policy: levels == false launches the plan, the leaves and every tree
// node's means; levels == true then the node states and versions.
cudaError_t launch_fenwick(const Dims &dm, const Plan &pl, const CallArgs &ca, float *treeS,
                           float *treeZ, bool bf16, bool levels, cudaStream_t s);
cudaError_t launch_readout_simt(const Dims &dm, const Plan &pl, const CallArgs &ca,
                                cudaStream_t s);
cudaError_t launch_decode_decide(const dla_cache &cc, float tau, int32_t dt, const void *q,
                                 const void *k, void *ws, uint8_t *boundary, int32_t *merge_i,
                                 int32_t *dev_status, cudaStream_t s,
                                 const uint8_t *active = nullptr);
cudaError_t launch_decode_stream(const dla_cache &cc, int32_t dt, const void *q, const void *k,
                                 const void *v, void *o, void *ws, cudaStream_t s);
size_t decode_ws_bytes(int32_t N, int32_t H, int32_t C);
size_t static_decode_max_bytes();
cudaError_t static_decode_scratch(void **out);

// Records a dla_profile event pair around one launch.
struct ProfScope {
  dla_profile *p;
  int idx;
  cudaStream_t s;
  ProfScope(dla_profile *prof, int kind, cudaStream_t st) : p(prof), idx(-1), s(st) {
    if (p && p->count < p->cap && p->begin && p->end) {
      idx = p->count;
      if (p->kind) p->kind[idx] = kind;
      cudaEventRecord(static_cast<cudaEvent_t>(p->begin[idx]), s);
    }
    if (p) p->count++;
  }
  ~ProfScope() {
    if (idx >= 0) cudaEventRecord(static_cast<cudaEvent_t>(p->end[idx]), s);
  }
};

}  // namespace dla
