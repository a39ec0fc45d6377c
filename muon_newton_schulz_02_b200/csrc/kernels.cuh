// Device kernels of the Muon step (Modded-NanoGPT article, "Muon optimizer"
// section: Nesterov momentum, then zeroth_power_via_newtonschulz5, then the
// weight update).
//
//   prologue_kernel   buf <- mu*buf + g ; G = g + mu*buf ; per-matrix ||G||_F ;
//                     X0 = bf16(G), stored short-side-major (k x l, padded).
//   ns_gemm_kernel    persistent tcgen05 GEMM over all matrices of a group,
//                     either one launch chaining every phase and the weight
//                     update (per-matrix completion counters order the
//                     phases), or one launch per phase:
//                       GRAM    A = s^2 * X X^T            (upper-triangle 256-blocks only)
//                       POLY    B' = a*I + b*A + c*(A A)   (upper-triangle 256-blocks only)
//                       UPDATE  X' = s*(B' X)              (last step: W -= lr*X')
//                     s = 1/(||G||_F+eps) on the first iteration, 1 afterwards,
//                     so the listing's normalisation is folded into epilogues;
//                     a*X + B X = (a*I + B) X, so the a*X term rides on the
//                     diagonal of B' and the update reads no second copy of X.
//                     (256 x 256 output tiles per cluster of two CTAs,
//                     tcgen05.mma.cta_group::2; a template per phase.)
//                     In the per-phase launches the A A and X X^T products of
//                     the first iterations may read e4m3 copies of their
//                     operands (kind::f8f6f4, muon_step_fp8).
//   ns_small_kernel   the whole step of a small matrix (short side <= 128,
//                     long side <= 512) in one CTA, everything on chip.
//   ns_pair_kernel    the same for 128 < short side <= 256, long side <= 256,
//                     on a cluster of two CTAs (cta_group::2 products).
//   o16_kernel        bf16 update exchange: O (fp32) -> bf16, or W -= lr * O.
//   apply_x0_kernel   ns_steps == 0: W -= lr * s * X0.
#pragma once

#include <cuda.h>
#include "ptx.cuh"

namespace muon {

constexpr int kTile = 256;          // pair tile: 256 x 256 outputs per CTA pair
constexpr int kBM = 128;            // rows of the pair tile held by one CTA (TMEM lanes)
constexpr int kBN = 256;            // columns of the pair tile (TMEM fp32 columns per accumulator)
constexpr int kBNh = 128;           // B-operand rows / columns loaded by one CTA (half of kBN)
constexpr int kBK = 64;             // K per pipeline stage: one 128-byte swizzle row of bf16
constexpr int kUmmaK = 16;          // K of one tcgen05.mma kind::f16
// The bounds-checking build (MUON_DEBUG_BOUNDS) checks every tile a GEMM role
// takes against its class, matrix and tile grid before touching memory for it;
// a tile outside them stops the launch with kDevBounds in the status word.
#ifdef MUON_DEBUG_BOUNDS
constexpr bool kBoundsChecks = true;
#else
constexpr bool kBoundsChecks = false;
#endif

constexpr int kStages = 5;          // operand stages of the per-phase launches
constexpr int kChainStages = 4;     // of the chained launch (measured faster there, slower per phase)
constexpr int kGemmThreads = 224;   // warp 0 TMA, warp 1 MMA (+TMEM alloc), warp 2 epilogue DMA, warps 3..6 epilogue math
constexpr int kEpiThreads = 128;
constexpr int kEpiWarp0 = 3;        // first epilogue math warp
constexpr int kTmemCols = 512;      // two 256-column fp32 accumulators
constexpr int kMaxClasses = 16;
constexpr int kMaxMats = 320;
constexpr int kTmapsPerClass = 8;
constexpr int kPad = 128;           // padding granule of the short and long sides
constexpr int kBK8 = 128;           // K per pipeline stage of e4m3 operands: one 128-byte swizzle row
constexpr int kUmmaK8 = 32;         // K of one tcgen05.mma kind::f8f6f4
constexpr int kTmaps8PerClass = 4;
constexpr int kMaxFp8Iters = 2;     // e4m3 operands reach at most the first two iterations
static_assert(kTile == 256 && kBK == 64 && kBK8 == 128, "K-block shifts in ns_gemm_kernel assume these sizes");

enum TmapSlot : int {
  kTmX0 = 0, kTmX1 = 1,             // iterates, 64 x 128 boxes (K-major operand rows, epilogue slices, stores)
  kTmX0mn = 2, kTmX1mn = 3,         // iterates, 64 x 64 boxes (MN-major operand of the update)
  kTmA = 4, kTmB = 5,               // Gram / polynomial matrices, 64 x 128 boxes
  kTmAmn = 6, kTmBmn = 7            // Gram / polynomial matrices, 64 x 64 boxes (transposed operand reads)
};
enum Tmap8Slot : int {
  kTm8X = 0, kTm8A = 1,             // e4m3 copies of X and A, 128 x 128 boxes (K-major and MN-major operand reads)
  kTm8Xs = 2, kTm8As = 3            // the same tensors, 64 x 128 boxes with the 64-byte swizzle (epilogue stores)
};
enum GemmMode : int { kModeGram = 0, kModePoly = 1, kModeUpdate = 2,
                      kModeFinal = 3 };   // work items only: the last update, with W -= lr*O

constexpr uint32_t kStageABytes = kBM * kBK * 2;     // 16 KB
constexpr uint32_t kStageBBytes = kBNh * kBK * 2;    // 16 KB
constexpr uint32_t kStageBytes = kStageABytes + kStageBBytes;
constexpr uint32_t kSliceBytes = kBM * 64 * 2;       // 16 KB: 128 rows x 64 cols bf16 (one TMA box)
constexpr uint32_t kSmemCtrlBytes = 512;
// dynamic shared memory of a GEMM launch with `stages` operand stages: the
// stages, the four 16 KB chunk buffers, the control block, alignment slack
constexpr uint32_t gemm_smem_bytes(int stages) {
  return stages * kStageBytes + 4 * kSliceBytes + kSmemCtrlBytes + 1024;
}
constexpr uint32_t kGemmSmemBytes = gemm_smem_bytes(kStages);
constexpr uint32_t kChainSmemBytes = gemm_smem_bytes(kChainStages);

// ------------------------------------------------------------ arguments ---
struct GemmClass {
  int batch;          // matrices of this shape class
  int kp, lp;         // padded short side (rows of X) and long side (cols of X)
  int mat_first;      // first matrix of the class in group order
  int tiles_m;        // ceil(kp / 256)
  int tiles_n;        // UPDATE: ceil(lp / 256); GRAM / POLY: tiles_m
  int tiles_per_mat;  // GRAM / POLY: tiles_m (tiles_m + 1) / 2; UPDATE: tiles_m * tiles_n
  int tile_begin;     // first tile of the class in this launch
  int kblocks;        // GRAM: lp / 64; POLY, UPDATE: kp / 64
  int tmap_base;      // first tensor map of the class in the table
};

struct OutMat {       // destination of the final UPDATE epilogue
  float* w;           // W (step) or O (orthogonalize), m x n row-major fp32
  int m, n;
  int trans;          // 1: X holds W^T (m > n)
  int vec;            // 1: n % 4 == 0 and w 16-byte aligned
  int tma;            // 1: wmaps[] holds a valid fp32 tensor map of w (needs vec)
};

// One unit of work of the chained launch: a 256 x 256 output tile of one
// phase (Gram, polynomial or update) of one Newton-Schulz iteration of one
// matrix.  The host lays out one list per cluster in an order in which every
// item's inputs are produced by items that come earlier in some list (see
// `need`), so the lists can run concurrently on all clusters.
struct WorkItem {
  int need;                 // tile halves of this matrix (2 per tile: one per CTA) that must have
                            // completed before this item reads its inputs
  unsigned short mat, b;    // matrix (group order), its index within its shape class
  unsigned short tm, tn;    // output tile row and column (256-blocks)
  unsigned char cls, mode;  // shape class, kModeGram / kModePoly / kModeUpdate / kModeFinal
  unsigned short it;        // Newton-Schulz iteration
};
static_assert(sizeof(WorkItem) == 16, "WorkItem layout");

struct GemmArgs {
  const CUtensorMap* tmaps;
  const CUtensorMap* tmaps8;  // per class kTmaps8PerClass maps of the e4m3 copies (null: no e4m3 iteration)
  const CUtensorMap* wmaps;   // per matrix (group order): W as fp32 [m][n]; box 32x128 (X = W) or 32x32 (X = W^T)
  const float* scale;     // per matrix (group order): 1/(||G||_F + eps)
  int* status;
  const WorkItem* items;  // chained launch: every cluster's work list, back to back
  const int* item_off;    // chained launch: cluster c runs items[item_off[c] .. item_off[c + 1])
  unsigned* done;         // chained launch: per matrix, tile halves completed (zeroed by the prologue)
  unsigned long long wait_limit_ns;
  int nclasses, total_tiles;
  int mode, x_in, first, final_apply, assign, debug_flags;
  int iter;               // one launch per phase: the Newton-Schulz iteration
  int fp8_iters;          // iterations whose products read e4m3 operands (see set_precision), <= kMaxFp8Iters
  float sx8[kMaxFp8Iters], sa8[kMaxFp8Iters];   // power-of-two scales of the e4m3 copies of X_i and A_i
  float a, b, c, lr;
  GemmClass cls[kMaxClasses];
  OutMat out[kMaxMats];
};

struct ProMat {
  const float* g;
  float* buf;
  __nv_bfloat16* x;   // padded kp x lp X0 of this matrix
  int m, n, kp, lp;
  int trans, vec;
  int tile_begin, tiles_c, tiles;
};

struct ProArgs {
  int nmats, total_tiles;
  float mu, eps;
  int nesterov, has_buf;
  float* partials;
  unsigned* tickets;
  float* scale;
  unsigned* done;         // per-matrix completion counters of the chained launch that follows (or null)
  ProMat mats[kMaxMats];
};

struct ApplyArgs {
  const float* scale;
  float lr;
  int assign, nmats;
  const __nv_bfloat16* x[kMaxMats];
  int lp[kMaxMats];
  OutMat out[kMaxMats];
};

// ============================================================ prologue ===
// One CTA per 64 x 128 tile of the padded X0 (short side k = rows of X).
constexpr int kProThreads = 256;
constexpr int kProRows = 64, kProCols = 128;

__device__ __forceinline__ int find_mat(const ProArgs& p, int t) {
  int lo = 0, hi = p.nmats - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (p.mats[mid].tile_begin <= t) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__device__ __forceinline__ float nesterov_g(float gv, float& bv, float mu, int nesterov, int has_buf) {
  if (!has_buf) return gv;
  bv = fmaf(mu, bv, gv);                    // buf <- mu*buf + g
  return nesterov ? fmaf(mu, bv, gv) : bv;  // G = g + mu*buf (new buf)
}

__global__ void __launch_bounds__(kProThreads) prologue_kernel(const __grid_constant__ ProArgs p) {
  __shared__ __align__(16) __nv_bfloat16 S[kProRows * kProCols];  // transposed path staging, 16B-unit swizzle
  __shared__ float red[kProThreads / 32];
  __shared__ unsigned last_flag;
  __shared__ double dred[kProThreads / 32];

  griddep_launch_dependents();
  griddep_wait();
  const int t = blockIdx.x;
  if (t == 0 && p.done)
    for (int i = threadIdx.x; i < p.nmats; i += kProThreads) p.done[i] = 0u;
  const int mi = find_mat(p, t);
  const ProMat& M = p.mats[mi];
  const int local = t - M.tile_begin;
  const int xr0 = (local / M.tiles_c) * kProRows;
  const int xc0 = (local % M.tiles_c) * kProCols;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  float ss = 0.f;

  if (!M.trans) {
    // X[xr][xc] = G[xr][xc]: each warp walks one row segment of 128 columns.
#pragma unroll
    for (int pass = 0; pass < kProRows / 8; ++pass) {
      const int row = xr0 + pass * 8 + warp;
      const int col = xc0 + lane * 4;
      float gv[4] = {0.f, 0.f, 0.f, 0.f}, bv[4] = {0.f, 0.f, 0.f, 0.f}, G[4] = {0.f, 0.f, 0.f, 0.f};
      const bool rok = row < M.m;
      const size_t off = (size_t)row * M.n + col;
      if (rok && M.vec) {
        if (col < M.n) {
          float4 g4 = __ldcs(reinterpret_cast<const float4*>(M.g + off));
          gv[0] = g4.x; gv[1] = g4.y; gv[2] = g4.z; gv[3] = g4.w;
          if (p.has_buf) {
            float4 b4 = __ldcs(reinterpret_cast<const float4*>(M.buf + off));
            bv[0] = b4.x; bv[1] = b4.y; bv[2] = b4.z; bv[3] = b4.w;
          }
#pragma unroll
          for (int q = 0; q < 4; ++q) G[q] = nesterov_g(gv[q], bv[q], p.mu, p.nesterov, p.has_buf);
          if (p.has_buf) __stcs(reinterpret_cast<float4*>(M.buf + off), make_float4(bv[0], bv[1], bv[2], bv[3]));
        }
      } else if (rok) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          if (col + q < M.n) {
            gv[q] = M.g[off + q];
            if (p.has_buf) bv[q] = M.buf[off + q];
            G[q] = nesterov_g(gv[q], bv[q], p.mu, p.nesterov, p.has_buf);
            if (p.has_buf) M.buf[off + q] = bv[q];
          }
        }
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) ss = fmaf(G[q], G[q], ss);
      uint2 packed = make_uint2(pack_bf16x2(G[0], G[1]), pack_bf16x2(G[2], G[3]));
      *reinterpret_cast<uint2*>(M.x + (size_t)row * M.lp + col) = packed;   // zero in the padding
    }
  } else {
    // X[xr][xc] = G[xc][xr]: read a 128 (G rows) x 64 (G cols) block, transpose in shared memory.
#pragma unroll
    for (int pass = 0; pass < kProCols / 16; ++pass) {
      const int gi_l = pass * 16 + (tid >> 4);      // 0..127: G row within block = X col
      const int gj_l = (tid & 15) * 4;              // 0..60 : G col within block = X row
      const int gi = xc0 + gi_l, gj = xr0 + gj_l;
      float gv[4] = {0.f, 0.f, 0.f, 0.f}, bv[4] = {0.f, 0.f, 0.f, 0.f}, G[4] = {0.f, 0.f, 0.f, 0.f};
      const bool rok = gi < M.m;
      const size_t off = (size_t)gi * M.n + gj;
      if (rok && M.vec) {
        if (gj < M.n) {
          float4 g4 = __ldcs(reinterpret_cast<const float4*>(M.g + off));
          gv[0] = g4.x; gv[1] = g4.y; gv[2] = g4.z; gv[3] = g4.w;
          if (p.has_buf) {
            float4 b4 = __ldcs(reinterpret_cast<const float4*>(M.buf + off));
            bv[0] = b4.x; bv[1] = b4.y; bv[2] = b4.z; bv[3] = b4.w;
          }
#pragma unroll
          for (int q = 0; q < 4; ++q) G[q] = nesterov_g(gv[q], bv[q], p.mu, p.nesterov, p.has_buf);
          if (p.has_buf) __stcs(reinterpret_cast<float4*>(M.buf + off), make_float4(bv[0], bv[1], bv[2], bv[3]));
        }
      } else if (rok) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          if (gj + q < M.n) {
            gv[q] = M.g[off + q];
            if (p.has_buf) bv[q] = M.buf[off + q];
            G[q] = nesterov_g(gv[q], bv[q], p.mu, p.nesterov, p.has_buf);
            if (p.has_buf) M.buf[off + q] = bv[q];
          }
        }
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        ss = fmaf(G[q], G[q], ss);
        const int r = gj_l + q;                          // X row within tile
        const int unit = (gi_l >> 3) ^ ((r >> 2) & 15);  // swizzled 16-byte unit
        S[r * kProCols + unit * 8 + (gi_l & 7)] = __float2bfloat16_rn(G[q]);
      }
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < (kProRows * kProCols / 8) / kProThreads; ++i) {
      const int chunk = tid + i * kProThreads;
      const int r = chunk >> 4, u = chunk & 15;
      const int su = u ^ ((r >> 2) & 15);
      uint4 v = *reinterpret_cast<const uint4*>(&S[r * kProCols + su * 8]);
      *reinterpret_cast<uint4*>(M.x + (size_t)(xr0 + r) * M.lp + xc0 + u * 8) = v;
    }
  }

  // Deterministic per-tile partial of ||G||_F^2, then the last tile of the
  // matrix sums all partials in tile order.
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if (lane == 0) red[warp] = ss;
  __syncthreads();
  if (tid == 0) {
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < kProThreads / 32; ++w) s += red[w];
    p.partials[t] = s;
    __threadfence();
    const unsigned ticket = atomicAdd(&p.tickets[mi], 1u);
    last_flag = (ticket == (unsigned)(M.tiles - 1));
  }
  __syncthreads();
  if (last_flag) {
    __threadfence();
    double acc = 0.0;
    for (int i = tid; i < M.tiles; i += kProThreads) acc += (double)__ldcg(&p.partials[M.tile_begin + i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) dred[warp] = acc;
    __syncthreads();
    if (tid == 0) {
      double tot = 0.0;
#pragma unroll
      for (int w = 0; w < kProThreads / 32; ++w) tot += dred[w];
      const float nrm = (float)sqrt(tot);
      p.scale[mi] = 1.0f / (nrm + p.eps);
      p.tickets[mi] = 0u;
    }
  }
}

// ====================================================== NS GEMM kernel ===
struct TileCoord { int cls, b, tm, tn; };

__device__ __forceinline__ TileCoord decode_tile(const GemmArgs& p, int t, bool sym) {
  int c = 0;
  while (c + 1 < p.nclasses && t >= p.cls[c + 1].tile_begin) ++c;
  const GemmClass& C = p.cls[c];
  const int local = t - C.tile_begin;
  TileCoord tc;
  tc.cls = c;
  tc.b = local / C.tiles_per_mat;
  int r = local - tc.b * C.tiles_per_mat;
  if (sym) {
    int tm = 0, rowlen = C.tiles_m;
    while (r >= rowlen) { r -= rowlen; ++tm; --rowlen; }
    tc.tm = tm;
    tc.tn = tm + r;
  } else {
    tc.tm = r / C.tiles_n;
    tc.tn = r - tc.tm * C.tiles_n;
  }
  return tc;
}

// One output tile as every role of the GEMM kernel sees it.
struct Tile {
  int mode;       // kModeGram / kModePoly / kModeUpdate
  int fin;        // the last update: the epilogue adds -lr*O into W
  int cls, b;     // shape class, matrix within the class
  int tm, tn;     // 256-block row and column of the output
  int x_in;       // which ping-pong iterate holds X (iteration parity)
  int first;      // first iteration: the normalisation scale is folded in
  int mat;        // matrix in group order
  int need;       // chained launch: tile halves of `mat` that must have completed first
  int it;         // Newton-Schulz iteration
  int op8;        // the product reads e4m3 copies of its operands (K = 128 per stage)
  int dual;       // besides its bf16 output, write the e4m3 copy the next product reads (A, or X)
  int nsub;       // chunks per 64-column slice of the output: 2 (last update, dual) or 1
};

// Which products of iteration `it` read e4m3 operands, for fp8_iters = F
// (0 <= F <= 2): the A A product of iterations 0 .. F-1 and the X X^T product
// of iterations 1 .. F-1.  The update B' X keeps bf16 operands throughout: an
// e4m3 rounding of the iterate itself moves its singular vectors, which no
// later iteration corrects, while a rounding of A only perturbs the polynomial
// that maps the singular values.  The first Gram product stays bf16 too: X0 is
// stored before the norm of G is known, so no fixed scale fits it, while every
// later iterate and Gram matrix is bounded through the singular values (see
// the host's scales).
// kFp8 = false (every launch of a bf16 step) compiles the e4m3 paths out.
template <bool kFp8>
__device__ __forceinline__ void set_precision(Tile& T, int F) {
  if constexpr (kFp8) {
    T.op8 = T.mode == kModePoly ? T.it < F : (T.mode == kModeGram && T.it >= 1 && T.it < F);
    T.dual = T.mode == kModeGram ? T.it < F : (T.mode == kModeUpdate && !T.fin && T.it + 1 < F);
  } else {
    T.op8 = 0;
    T.dual = 0;
  }
  T.nsub = (T.fin || T.dual) ? 2 : 1;
}

// Byte offset of the 16-byte unit u (0..7) of row r inside a 128-row x 128-byte
// box stored with the 128-byte swizzle (the pattern TMA writes / reads).
__device__ __forceinline__ uint32_t sw128_off(uint32_t r, uint32_t u) { return r * 128u + ((u ^ (r & 7u)) << 4); }

// Read-modify-write of this warp's 32 rows of a 128 x 32 slice of the final
// result into W (or O), for outputs whose rows are not 16-byte aligned.  The
// slice is staged in shared memory by the same warp (rows 32q..32q+31); X row
// gi0 + r, col gj0 + c maps to W[gi][gj] (X = W) or W[gj][gi] (X = W^T).  Every
// access pattern touches whole 128-byte rows of W.
__device__ __forceinline__ void store_w_slice_warp(const OutMat& O, const float* S, int gi0, int gj0, int q,
                                                   int lane, float lr, int assign) {
  if (!O.trans) {
#pragma unroll 2
    for (int it = 0; it < 8; ++it) {
      const int rr = q * 32 + it * 4 + (lane >> 3), qd = lane & 7;
      const int gi = gi0 + rr, gj = gj0 + 4 * qd;
      if (gi >= O.m || gj >= O.n) continue;
      const float4 o = *reinterpret_cast<const float4*>(S + rr * 32 + ((qd ^ (rr & 7)) << 2));
      float* wp = O.w + (size_t)gi * O.n + gj;
      const float ov[4] = {o.x, o.y, o.z, o.w};
      for (int e = 0; e < 4 && gj + e < O.n; ++e) wp[e] = assign ? ov[e] : wp[e] - lr * ov[e];
    }
  } else {
    const int wcol = gi0 + q * 32 + lane;           // W column = X row
#pragma unroll 4
    for (int c = 0; c < 32; ++c) {
      const int wrow = gj0 + c;                      // W row = X column
      if (wrow >= O.m || wcol >= O.n) continue;
      const float o = S[c * kBM + q * 32 + lane];
      float* wp = O.w + (size_t)wrow * O.n + wcol;
      *wp = assign ? o : *wp - lr * o;
    }
  }
}

struct __align__(8) GemmCtrl {
  uint64_t full[kStages];     // even CTA: both CTAs' operand bytes of a stage have landed
  uint64_t empty[kStages];    // the pair MMAs reading a stage are done (both CTAs)
  uint64_t tmem_full[2];      // an accumulator is ready (both CTAs)
  uint64_t tmem_empty[2];     // even CTA: all 8 epilogue math warps of the pair drained an accumulator
  uint64_t in_full[4];        // DMA -> math: chunk buffer handed over (its input slice landed, if any)
  uint64_t out_full[4];       // math -> DMA: chunk staged (and its input consumed)
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  int prod_passed;            // chained launch: items whose inputs the producer has seen complete
};
static_assert(sizeof(GemmCtrl) <= kSmemCtrlBytes, "GemmCtrl does not fit its shared-memory slot");
static_assert(kGemmSmemBytes <= 232448 && kChainSmemBytes <= 232448, "more dynamic shared memory than a CTA may have");
static_assert(kChainStages <= kStages, "GemmCtrl holds kStages barriers per ring");

// The Newton-Schulz GEMM kernel.  A cluster of two CTAs (one per SM) computes
// 256 x 256 output tiles with tcgen05.mma.cta_group::2: each CTA loads its 128
// rows of A and its 128 rows (or columns) of B per stage, the even CTA issues
// the MMAs over both CTAs' shared memory, and each CTA's TMEM holds its 128
// rows x 256 fp32 columns (two accumulators, double-buffered).  Roles per CTA:
// warp 0 TMA producer; warp 1 MMA issuer (even CTA) and TMEM allocator; warp 2
// epilogue DMA (loads the polynomial epilogue's A slices, issues the TMA
// stores / add-reductions of the output and recycles their buffers); warps
// 3..6 epilogue math (tcgen05.ld -> fp32 math -> bf16 or fp32 -> 128B-swizzled
// smem).  The math warps hand output chunks to the DMA warp through a ring of
// four 16 KB buffers and mbarriers, and never wait on TMA latency themselves:
// an ordinary tile is 4 chunks (bf16 64-column slices), a tile of the last
// update 8 chunks (fp32 32-column halves of a slice, added into W in L2).
//
// Two ways to launch it:
//   kChain = false: one launch per phase (kMode) over all matrices of a group,
//     persistent, tile t to cluster t mod #clusters; kFinal selects the last
//     update, whose epilogue adds -lr*O into W.
//   kChain = true: one launch for every phase of every iteration.  Each
//     cluster runs its own list of work items (any phase, any matrix; the host
//     orders the lists so that items are ready in time); before reading a
//     matrix's Gram, polynomial or iterate it waits (bounded) for the counter
//     of completed tiles of that matrix, and after its output stores have
//     landed it adds one to that counter.  A matrix's phases then follow each
//     other closely on whichever clusters are free, without a launch
//     boundary, its operands are still in L2 when they are read, and the
//     weight update of one matrix overlaps the products of others.
template <int kMode, bool kFinal, bool kChain, bool kFp8 = false>
__global__ void __launch_bounds__(kGemmThreads, 1) ns_gemm_kernel(const __grid_constant__ GemmArgs p) {
  static_assert(!(kChain && kFinal), "the chained launch takes the final update from its items");
  static_assert(!(kChain && kFp8), "e4m3 operands run only in the per-phase launches");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stage_base = smem;
  constexpr int kSt = kChain ? kChainStages : kStages;
  uint8_t* dbuf = smem + kSt * kStageBytes;            // 2 x 16 KB: slice buffers 0, 1 / fp32 staging 2, 3
  uint8_t* mbuf = dbuf + 2 * kSliceBytes;              // 2 x 16 KB: slice buffers 2, 3 / fp32 staging 0, 1
  GemmCtrl* ctl = reinterpret_cast<GemmCtrl*>(mbuf + 2 * kSliceBytes);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();             // 0: issues the MMAs of the pair
  const int cid = (int)cluster_id_x(), ncl = (int)cluster_count_x();
  // The ring of four 16 KB chunk buffers: running chunk q uses buffer q % 4.
  auto slice_buf = [&](int b) { return b < 2 ? dbuf + b * kSliceBytes : mbuf + (b - 2) * kSliceBytes; };

  // This cluster's tiles, in processing order.
  const int item0 = kChain ? p.item_off[cid] : 0;
  const int my_tiles = kChain ? p.item_off[cid + 1] - item0
                              : (cid < p.total_tiles ? (p.total_tiles - cid + ncl - 1) / ncl : 0);
  auto tile_of = [&](int i) {
    Tile T;
    if constexpr (kChain) {
      const WorkItem w = p.items[item0 + i];
      T.fin = w.mode == kModeFinal;
      T.mode = T.fin ? kModeUpdate : w.mode; T.cls = w.cls; T.b = w.b; T.tm = w.tm; T.tn = w.tn;
      T.x_in = w.it & 1; T.first = w.it == 0; T.mat = w.mat; T.need = w.need; T.it = w.it;
    } else {
      const TileCoord tc = decode_tile(p, cid + i * ncl, kMode != kModeUpdate);
      T.mode = kMode; T.fin = kFinal; T.cls = tc.cls; T.b = tc.b; T.tm = tc.tm; T.tn = tc.tn;
      T.x_in = p.x_in; T.first = p.first; T.mat = p.cls[tc.cls].mat_first + tc.b; T.need = 0; T.it = p.iter;
    }
    set_precision<kFp8>(T, p.fp8_iters);
    return T;
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < kSt; ++s) { mbar_init(&ctl->full[s], 1); mbar_init(&ctl->empty[s], 1); }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&ctl->tmem_full[s], 1);
      mbar_init(&ctl->tmem_empty[s], 8);
    }
    for (int s = 0; s < 4; ++s) {
      mbar_init(&ctl->in_full[s], 1);
      mbar_init(&ctl->out_full[s], 4);
    }
    mbar_init(&ctl->drain, 1);
    ctl->abort_flag = 0;
    ctl->prod_passed = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(&ctl->tmem_base, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();                                  // barriers of both CTAs initialised
  tc_fence_after();
  const uint32_t tmem_base = ctl->tmem_base;
  WaitCtx wc{&ctl->abort_flag, p.status, p.wait_limit_ns, mapa_shared(&ctl->abort_flag, rank ^ 1u)};
  bool aborted = false;
  // bounds-checking build: a tile outside its class's matrices and tile grid
  auto out_of_range = [&](const Tile& T) {
    if constexpr (!kBoundsChecks) {
      return false;
    } else {
      bool in = T.cls >= 0 && T.cls < p.nclasses;
      if (in) {
        const GemmClass& C = p.cls[T.cls];
        const int tiles_k = (C.kp + kTile - 1) / kTile, tiles_l = (C.lp + kTile - 1) / kTile;
        in = T.b >= 0 && T.b < C.batch && T.mat == C.mat_first + T.b && T.mat < kMaxMats && T.tm >= 0 &&
             T.tm < tiles_k && T.tn >= 0 && T.tn < (T.mode == kModeUpdate ? tiles_l : tiles_k) &&
             (T.mode == kModeUpdate || T.tm <= T.tn);
      }
      if (!in) raise_error(wc, kDevBounds);
      return !in;
    }
  };
  // set-up above overlaps the previous launch; its outputs are read only below
  griddep_launch_dependents();
  griddep_wait();

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    if (lane == 0) {
      for (int c = 0; c < p.nclasses; ++c)
        for (int k = 0; k < kTmapsPerClass; ++k) {
          const CUtensorMap* tm = &p.tmaps[p.cls[c].tmap_base + k];
          tmap_acquire(tm);
          tmap_prefetch(tm);
        }
      if (kFp8 && p.tmaps8)
        for (int c = 0; c < p.nclasses; ++c)
          for (int k = kTm8X; k <= kTm8A; ++k) {
            const CUtensorMap* tm = &p.tmaps8[c * kTmaps8PerClass + k];
            tmap_acquire(tm);
            tmap_prefetch(tm);
          }
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int it = 0; it < my_tiles && ok; ++it) {
        const Tile T = tile_of(it);
        if (out_of_range(T)) { ok = false; break; }
        const GemmClass& C = p.cls[T.cls];
        const bool sym = T.mode != kModeUpdate;
        if (kChain && T.need > 0) {
          // this tile reads what earlier tiles of the matrix wrote
          if (!wait_count(&p.done[T.mat], (uint32_t)T.need, wc, kDevTimeoutDep)) { ok = false; break; }
          fence_proxy_async_global();
        }
        if (kChain) st_release_cta_shared(&ctl->prod_passed, it + 1);   // inputs of items 0..it are complete
        const CUtensorMap* tA;
        const CUtensorMap* tB;
        if (T.mode == kModeGram) { tA = &p.tmaps[C.tmap_base + (T.x_in ? kTmX1 : kTmX0)]; tB = tA; }
        else if (T.mode == kModePoly) { tA = &p.tmaps[C.tmap_base + kTmA]; tB = tA; }
        else { tA = &p.tmaps[C.tmap_base + kTmB]; tB = &p.tmaps[C.tmap_base + (T.x_in ? kTmX1mn : kTmX0mn)]; }
        const int arow = T.tm * kTile + (int)rank * kBM;     // this CTA's A rows
        const int bidx = T.tn * kTile + (int)rank * kBNh;    // this CTA's B rows (or columns)
        // The Gram and polynomial matrices hold only their upper-triangle 256-blocks:
        // an operand block below the diagonal is read through its stored transpose.
        const CUtensorMap* tAt = (T.mode == kModePoly) ? &p.tmaps[C.tmap_base + kTmAmn]
                                                       : &p.tmaps[C.tmap_base + kTmBmn];
        // e4m3 operands (Gram: X, polynomial: A): one 128 x 128 box per operand and
        // stage, read K-major or (blocks below the diagonal) MN-major from one map
        const CUtensorMap* t8 = T.op8 ? &p.tmaps8[T.cls * kTmaps8PerClass + (T.mode == kModeGram ? kTm8X : kTm8A)]
                                      : nullptr;
        const int kbsh = T.op8 ? 1 : 2;                       // K-block kb lies in 256-block kb >> kbsh
        const int kblocks = (T.mode == kModeGram ? C.lp : C.kp) >> (8 - kbsh);
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(&ctl->empty[stage], phase ^ 1u, wc, kDevTimeoutEmpty)) { ok = false; break; }
          uint8_t* sa = stage_base + stage * kStageBytes;
          uint8_t* sb = sa + kStageABytes;
          const uint32_t full_lead = mapa_shared(&ctl->full[stage], 0);
          const bool inject_skip = (p.debug_flags & 1) && it == 0 && kb == 0;
          // on a diagonal tile of the symmetric phases a CTA's A rows are its B
          // rows: load them once, the MMA reads both operands from the A buffer
          const bool same_ab = sym && T.tm == T.tn;
          const bool a_below = T.mode != kModeGram && T.tm > (kb >> kbsh);
          const bool b_mn = T.mode == kModeUpdate || (T.mode == kModePoly && T.tn > (kb >> kbsh));
          if (!inject_skip && T.op8) {
            if (rank == 0) mbar_arrive_expect_tx(&ctl->full[stage], same_ab ? 2 * kStageABytes : 2 * kStageBytes);
            if (a_below) tma_load_3d_pair(sa, t8, full_lead, arow, kb * kBK8, T.b);
            else tma_load_3d_pair(sa, t8, full_lead, kb * kBK8, arow, T.b);
            if (!same_ab) {
              if (b_mn) tma_load_3d_pair(sb, t8, full_lead, bidx, kb * kBK8, T.b);
              else tma_load_3d_pair(sb, t8, full_lead, kb * kBK8, bidx, T.b);
            }
          } else if (!inject_skip) {
            if (rank == 0) mbar_arrive_expect_tx(&ctl->full[stage], same_ab ? 2 * kStageABytes : 2 * kStageBytes);
            if (a_below) {
              // A rows below the diagonal block: columns [arow, +128) of rows [kb*64, +64), MN-major
              tma_load_3d_pair(sa, tAt, full_lead, arow, kb * kBK, T.b);
              tma_load_3d_pair(sa + kStageABytes / 2, tAt, full_lead, arow + 64, kb * kBK, T.b);
            } else {
              tma_load_3d_pair(sa, tA, full_lead, kb * kBK, arow, T.b);
            }
            if (same_ab) {
              // nothing: B is the A block just loaded
            } else if (b_mn) {
              // B = rows [kb*64, +64) x this CTA's 128 columns, MN-major: two 64-col boxes
              const CUtensorMap* tBm = (T.mode == kModeUpdate) ? tB : tAt;
              tma_load_3d_pair(sb, tBm, full_lead, bidx, kb * kBK, T.b);
              tma_load_3d_pair(sb + kStageBBytes / 2, tBm, full_lead, bidx + 64, kb * kBK, T.b);
            } else {
              tma_load_3d_pair(sb, tB, full_lead, kb * kBK, bidx, T.b);
            }
          }
          if (++stage == kSt) { stage = 0; phase ^= 1u; }
        }
      }
      aborted = !ok;
    }
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA issuer
    if (lane == 0 && rank == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      bool issued_any = false;
      for (int it = 0; it < my_tiles && ok; ++it) {
        const Tile T = tile_of(it);
        if (out_of_range(T)) { ok = false; break; }
        const GemmClass& C = p.cls[T.cls];
        const bool sym = T.mode != kModeUpdate;
        const int acc = it & 1;
        const uint32_t acc_phase = (uint32_t)((it >> 1) & 1);
        if (!mbar_wait_cluster(&ctl->tmem_empty[acc], acc_phase ^ 1u, wc, kDevTimeoutAccum)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * kBN);
        const int kbsh = T.op8 ? 1 : 2;
        const int kblocks = (T.mode == kModeGram ? C.lp : C.kp) >> (8 - kbsh);
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(&ctl->full[stage], phase, wc, kDevTimeoutFull)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_u32(stage_base + stage * kStageBytes);
          // same choices as the producer: diagonal tiles of the symmetric phases
          // share one operand buffer, blocks below the diagonal arrive MN-major
          const bool same_ab = sym && T.tm == T.tn;
          const uint32_t sb = same_ab ? sa : sa + kStageABytes;
          const uint32_t a_mn = (T.mode != kModeGram && T.tm > (kb >> kbsh)) ? 1u : 0u;
          const uint32_t b_mn = same_ab ? a_mn
                                : (T.mode == kModeUpdate || (T.mode == kModePoly && T.tn > (kb >> kbsh))) ? 1u : 0u;
          if (T.op8) {
            // 128 MN bytes per CTA: one swizzle atom wide, so only the K stride (SBO) matters MN-major
            const uint32_t idesc = idesc_e4m3_f32(2 * kBM, kBN, a_mn, b_mn);
#pragma unroll
            for (int kk = 0; kk < kBK8 / kUmmaK8; ++kk) {
              const uint64_t adesc = a_mn ? smem_desc_sw128(sa + kk * (kUmmaK8 * 128), kStageABytes, 1024)
                                          : smem_desc_sw128(sa + kk * kUmmaK8, 16, 1024);
              const uint64_t bdesc = b_mn ? smem_desc_sw128(sb + kk * (kUmmaK8 * 128), kStageBBytes, 1024)
                                          : smem_desc_sw128(sb + kk * kUmmaK8, 16, 1024);
              tc_mma_e4m3_pair(d_tmem, adesc, bdesc, idesc, (kb | kk) != 0 ? 1u : 0u);
            }
          } else {
            const uint32_t idesc = idesc_bf16_f32(2 * kBM, kBN, a_mn, b_mn);
#pragma unroll
            for (int kk = 0; kk < kBK / kUmmaK; ++kk) {
              const uint64_t adesc = a_mn ? smem_desc_sw128(sa + kk * (kUmmaK * 128), kStageABytes / 2, 1024)
                                          : smem_desc_sw128(sa + kk * (kUmmaK * 2), 16, 1024);
              const uint64_t bdesc = b_mn ? smem_desc_sw128(sb + kk * (kUmmaK * 128), kStageBBytes / 2, 1024)
                                          : smem_desc_sw128(sb + kk * (kUmmaK * 2), 16, 1024);
              tc_mma_bf16_pair(d_tmem, adesc, bdesc, idesc, (kb | kk) != 0 ? 1u : 0u);
            }
          }
          issued_any = true;
          tc_commit_pair(mapa_shared(&ctl->empty[stage], 0));
          tc_commit_pair(mapa_shared(&ctl->empty[stage], 1));
          if (++stage == kSt) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        tc_commit_pair(mapa_shared(&ctl->tmem_full[acc], 0));
        tc_commit_pair(mapa_shared(&ctl->tmem_full[acc], 1));
      }
      if (issued_any) {                 // all MMAs done before TMEM is released
        tc_commit_pair(mapa_shared(&ctl->drain, 0));
        mbar_wait(&ctl->drain, 0, wc, kDevTimeoutDrain);
      }
      aborted = !ok;
    }
  } else if (warp == 2) {
    // ----------------------------------------------------- epilogue DMA
    if (lane == 0) {
      for (int c = 0; c < p.nclasses; ++c)
        for (int k = 0; k < kTmapsPerClass; ++k) tmap_acquire(&p.tmaps[p.cls[c].tmap_base + k]);
      if (kFp8 && p.tmaps8)
        for (int c = 0; c < p.nclasses; ++c)
          for (int k = kTm8Xs; k <= kTm8As; ++k) tmap_acquire(&p.tmaps8[c * kTmaps8PerClass + k]);
      if (p.final_apply)
        for (int c = 0; c < p.nclasses; ++c)
          for (int b = 0; b < p.cls[c].batch; ++b)
            if (p.out[p.cls[c].mat_first + b].tma) tmap_acquire(&p.wmaps[p.cls[c].mat_first + b]);
      int pend[4] = {-1, -1, -1, -1};              // parity of an input load not yet seen landed
      bool ok = true;
      // Arming chunk q hands buffer q % 4 to the math warps: with the A block
      // the polynomial epilogue adds loaded into it, or empty.  In the chained
      // launch a polynomial tile's chunks are armed only once its inputs are
      // known to be complete -- the producer has passed the tile's dependency
      // wait -- or once the DMA has reached that tile, after every earlier
      // tile published its results; so waiting there for the tile's inputs
      // never waits on this cluster, and the A slices usually load while the
      // previous tile is still draining.
      int ia = 0, ha = 0, armed = 0;               // next chunk to arm: chunk ha of tile ia
      Tile TA{};
      if (my_tiles > 0) TA = tile_of(0);
      auto deferred = [&](int drain_tile) {
        return kChain && ia < my_tiles && TA.mode == kModePoly && ia != drain_tile &&
               ld_acquire_cta_shared(&ctl->prod_passed) <= ia;
      };
      auto arm_until = [&](int limit, int drain_tile) {
        while (ok && armed < limit && ia < my_tiles && !deferred(drain_tile)) {
          if (out_of_range(TA)) { ok = false; return; }
          const int b = armed & 3;
          if (TA.mode == kModePoly) {
            if (kChain && ha == 0 && TA.need > 0) {
              ok = wait_count(&p.done[TA.mat], (uint32_t)TA.need, wc, kDevTimeoutDep);
              fence_proxy_async_global();
              if (!ok) return;
            }
            const GemmClass& C = p.cls[TA.cls];
            mbar_arrive_expect_tx(&ctl->in_full[b], kSliceBytes);
            tma_load_3d(slice_buf(b), &p.tmaps[C.tmap_base + kTmA], &ctl->in_full[b], TA.tn * kTile + 64 * ha,
                        TA.tm * kTile + (int)rank * kBM, TA.b);
            pend[b] = (armed >> 2) & 1;
          } else {
            mbar_arrive(&ctl->in_full[b]);
          }
          ++armed;
          if (++ha == 4 * TA.nsub) {
            ha = 0;
            if (++ia < my_tiles) TA = tile_of(ia);
          }
        }
      };
      arm_until(4, 0);
      int q = 0;                                   // next chunk to drain
      for (int i = 0; i < my_tiles && ok; ++i) {
        const Tile T = tile_of(i);
        if (out_of_range(T)) { ok = false; break; }
        const GemmClass& C = p.cls[T.cls];
        const int row0 = T.tm * kTile + (int)rank * kBM;
        const int nch = 4 * T.nsub;
        const CUtensorMap* tO = T.mode == kModeGram ? &p.tmaps[C.tmap_base + kTmA]
                              : T.mode == kModePoly ? &p.tmaps[C.tmap_base + kTmB]
                                                    : &p.tmaps[C.tmap_base + (T.x_in ? kTmX0 : kTmX1)];
        // e4m3 copy of the output (dual tiles): of A (Gram) or of the next iterate (update)
        const CUtensorMap* tO8 = !T.dual ? nullptr
                               : &p.tmaps8[T.cls * kTmaps8PerClass + (T.mode == kModeGram ? kTm8As : kTm8Xs)];
        for (int h = 0; h < nch; ++h, ++q) {
          const int b = q & 3;
          if (!mbar_wait(&ctl->out_full[b], (uint32_t)((q >> 2) & 1), wc, kDevTimeoutEpi)) { ok = false; break; }
          pend[b] = -1;                            // the math warps saw this chunk's input land
          const uint8_t* S = slice_buf(b);
          if (T.fin) {
            // -lr*O chunk: columns gj0..gj0+31 of X rows row0..row0+127
            const OutMat& O = p.out[T.mat];
            if (O.tma) {
              const CUtensorMap* wm = &p.wmaps[T.mat];
              const int gj0 = T.tn * kTile + 64 * (h >> 1) + 32 * (h & 1);
              if (!O.trans) {
                if (row0 < O.m && gj0 < O.n) {
                  if (p.assign) tma_store_2d(wm, S, gj0, row0); else tma_reduce_add_2d(wm, S, gj0, row0);
                }
              } else if (gj0 < O.m) {
                for (int hq = 0; hq < 4; ++hq) {
                  if (row0 + 32 * hq >= O.n) continue;
                  if (p.assign) tma_store_2d(wm, S + hq * 4096, row0 + 32 * hq, gj0);
                  else tma_reduce_add_2d(wm, S + hq * 4096, row0 + 32 * hq, gj0);
                }
              }
            }                                      // (rows not 16-byte aligned: the math warps wrote W)
          } else {
            // stores start inside the tensor only (a pair tile can overhang the
            // 128-padded edge by half; the overhang is never stored)
            const int ocols = T.mode != kModeUpdate ? C.kp : C.lp;
            const int x0 = T.tn * kTile + 64 * (h / T.nsub);
            const CUtensorMap* dst = (T.dual && (h & 1)) ? tO8 : tO;   // a dual tile's odd chunks: the e4m3 copy
            if (row0 < C.kp && x0 < ocols) tma_store_3d(dst, S, x0, row0, T.b);
          }
          tma_store_commit();                      // one bulk group per chunk
          if (armed < q + 4 && ia < my_tiles && !deferred(i)) {
            tma_store_wait_read1();                // the previous chunk's buffer has been read
            arm_until(q + 4, i);
          }
        }
        if (!ok) break;
        if (kChain && !T.fin) {
          tma_store_wait_all0();                   // this tile's output has landed in memory
          fence_proxy_async_global();
          red_release_gpu_add(&p.done[T.mat], 1u);
        }
        if (armed < q + 3 && ia < my_tiles) {      // chunks held back until this tile was published
          tma_store_wait_all0();
          arm_until(q + 4, i + 1);
        }
      }
      tma_store_wait_all0();
      for (int b = 0; b < 4; ++b)
        if (pend[b] >= 0) mbar_wait(&ctl->in_full[b], (uint32_t)pend[b], wc, kDevTimeoutDrain);
      aborted = !ok;
    }
  } else {
    // ---------------------------------------------------- epilogue math
    const int q4 = warp & 3;                      // TMEM lane quarter this warp may access
    const int r = q4 * 32 + lane;                 // tile row owned by this thread
    int q = 0;                                    // running chunk
    bool ok = true;
    // waits until chunk q's buffer is handed over (and its input, if any, landed)
    auto take = [&]() {
      return __all_sync(0xffffffffu, mbar_wait(&ctl->in_full[q & 3], (uint32_t)((q >> 2) & 1), wc, kDevTimeoutEpi));
    };
    for (int it = 0; it < my_tiles && ok; ++it) {
      const Tile T = tile_of(it);
      if (out_of_range(T)) { ok = false; break; }
      const int acc = it & 1;
      const uint32_t acc_phase = (uint32_t)((it >> 1) & 1);
      ok = __all_sync(0xffffffffu, mbar_wait(&ctl->tmem_full[acc], acc_phase, wc, kDevTimeoutAccum));
      if (!ok) break;
      tc_fence_after();
      const float s = T.first ? p.scale[T.mat] : 1.0f;
      // an e4m3 product carries the (power-of-two) scales of its operand copies
      const float pscale = !T.op8 ? 1.f
                           : T.mode == kModeGram ? 1.f / (p.sx8[T.it] * p.sx8[T.it])
                                                 : 1.f / (p.sa8[T.it] * p.sa8[T.it]);
      // scale of this tile's e4m3 output copy
      const float oscale = !T.dual ? 1.f : T.mode == kModeGram ? p.sa8[T.it] : p.sx8[T.it + 1];
      const int row0 = T.tm * kTile + (int)rank * kBM;
      const uint32_t tbase = tmem_base + ((uint32_t)(q4 * 32) << 16) + (uint32_t)(acc * kBN);
#pragma unroll 1
      for (int h = 0; h < 4 && ok; ++h) {
        if (!T.fin && !(ok = take())) break;
        float v[64];
        tmem_ld_32x32b_x64(tbase + (uint32_t)(h * 64), v);
        if (h == 3) {                               // accumulator fully read: hand it back to the MMA
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(mapa_shared(&ctl->tmem_empty[acc], 0));
        }
        if (T.mode != kModePoly) {
          // Gram: s^2 X X^T.  Update: s (aI + B) X = a s X + s B X, the aI term
          // carried on the diagonal of the polynomial phase's output.
          const float alpha = (T.mode == kModeGram ? s * s : s) * pscale;
#pragma unroll
          for (int i = 0; i < 64; ++i) v[i] *= alpha;
        } else {
          // b A + c A A
          const float cm = p.c * pscale;
          const uint8_t* dslice = slice_buf(q & 3);
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            uint4 raw = *reinterpret_cast<const uint4*>(dslice + sw128_off((uint32_t)r, (uint32_t)u));
            const __nv_bfloat162* hv = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              float2 f = __bfloat1622float2(hv[e]);
              v[u * 8 + 2 * e] = fmaf(cm, v[u * 8 + 2 * e], p.b * f.x);
              v[u * 8 + 2 * e + 1] = fmaf(cm, v[u * 8 + 2 * e + 1], p.b * f.y);
            }
          }
          // + a on the diagonal: on a diagonal tile, a warp's 32 rows meet the
          // slice's columns at 32 consecutive columns starting at dbase, lane by lane
          const int dbase = (int)rank * kBM + q4 * 32 - 64 * h;
          if (T.tm == T.tn && (dbase == 0 || dbase == 32)) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              if (j == lane) {
                if (dbase == 0) v[j] += p.a; else v[32 + j] += p.a;
              }
            }
          }
        }
        if (T.fin) {
          const OutMat& O = p.out[T.mat];
#pragma unroll
          for (int sub = 0; sub < 2; ++sub) {
            if (!(ok = take())) break;
            uint8_t* S = slice_buf(q & 3);
            const float* vv = v + 32 * sub;
            if (O.tma) {
              // -lr*O (or O), 128-byte swizzled; the DMA warp adds it to W in L2
              const float sg = p.assign ? 1.f : -p.lr;
              if (!O.trans) {
#pragma unroll
                for (int j = 0; j < 8; ++j)
                  *reinterpret_cast<float4*>(S + sw128_off((uint32_t)r, (uint32_t)j)) =
                      make_float4(sg * vv[4 * j], sg * vv[4 * j + 1], sg * vv[4 * j + 2], sg * vv[4 * j + 3]);
              } else {
                // box r / 32 holds W rows gj0..gj0+31 x W cols row0+32*(r/32)..+31
                uint8_t* Sh = S + (r >> 5) * 4096;
                const int rr = r & 31;
#pragma unroll
                for (int i = 0; i < 32; ++i)
                  *reinterpret_cast<float*>(Sh + sw128_off((uint32_t)i, (uint32_t)(rr >> 2)) + (rr & 3) * 4) =
                      sg * vv[i];
              }
              fence_async_shared();
            } else {
              // rows not 16-byte aligned: the math warps update W themselves,
              // in whole 128-byte rows through the chunk buffer
              float* Sf = reinterpret_cast<float*>(S);
              if (!O.trans) {
#pragma unroll
                for (int j = 0; j < 8; ++j)
                  *reinterpret_cast<float4*>(Sf + r * 32 + ((j ^ (r & 7)) << 2)) =
                      make_float4(vv[4 * j], vv[4 * j + 1], vv[4 * j + 2], vv[4 * j + 3]);
              } else {
#pragma unroll
                for (int i = 0; i < 32; ++i) Sf[i * kBM + r] = vv[i];
              }
              __syncwarp();
              store_w_slice_warp(O, Sf, row0, T.tn * kTile + 64 * h + 32 * sub, q4, lane, p.lr, p.assign);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&ctl->out_full[q & 3]);
            ++q;
          }
        } else {
          // bf16 output (in place over the input slice), 128-byte swizzled for the TMA store
          uint8_t* dslice = slice_buf(q & 3);
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            uint4 o;
            o.x = pack_bf16x2(v[u * 8 + 0], v[u * 8 + 1]);
            o.y = pack_bf16x2(v[u * 8 + 2], v[u * 8 + 3]);
            o.z = pack_bf16x2(v[u * 8 + 4], v[u * 8 + 5]);
            o.w = pack_bf16x2(v[u * 8 + 6], v[u * 8 + 7]);
            *reinterpret_cast<uint4*>(dslice + sw128_off((uint32_t)r, (uint32_t)u)) = o;
          }
          if (T.dual) {
            // the e4m3 copy goes into the next chunk: 128 rows x 64 bytes with the
            // 64-byte swizzle (16-byte unit u of row r at unit u ^ ((r >> 1) & 3))
            fence_async_shared();
            __syncwarp();
            if (lane == 0) mbar_arrive(&ctl->out_full[q & 3]);
            ++q;
            if (!(ok = take())) break;
            dslice = slice_buf(q & 3);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const float* w = v + 16 * u;
              uint4 o;
              o.x = pack_e4m3x4(oscale * w[0], oscale * w[1], oscale * w[2], oscale * w[3]);
              o.y = pack_e4m3x4(oscale * w[4], oscale * w[5], oscale * w[6], oscale * w[7]);
              o.z = pack_e4m3x4(oscale * w[8], oscale * w[9], oscale * w[10], oscale * w[11]);
              o.w = pack_e4m3x4(oscale * w[12], oscale * w[13], oscale * w[14], oscale * w[15]);
              *reinterpret_cast<uint4*>(dslice + r * 64 + ((u ^ ((r >> 1) & 3)) << 4)) = o;
            }
          }
          fence_async_shared();
          __syncwarp();
          if (lane == 0) mbar_arrive(&ctl->out_full[q & 3]);
          ++q;
        }
      }
    }
    aborted = !ok;
  }

  // On the abort path, give copies that a CTA issued towards its shared memory
  // time to land before either CTA of the pair leaves (bounded).
  if (aborted || *reinterpret_cast<volatile int*>(&ctl->abort_flag)) sleep_ns_bounded(200000);
  tc_fence_before();
  cluster_sync_all();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

// ================================================ small matrices, fused ===
// The whole step of one small matrix (short side k <= 128, long side l <= 512)
// in one CTA: momentum and norm while X0 is written into shared memory, then
// every quintic iteration with X, A and B resident in shared memory and the
// accumulators in TMEM, then the apply.  One launch covers every small matrix
// of a call (one CTA each).  X is stored as 128-row x 64-column chunks with
// the 128-byte swizzle: read K-major by the Gram product and MN-major (LBO =
// chunk stride) by the update, so it is never transposed.
constexpr int kSmallThreads = 128;
constexpr int kSmallMaxK = 128;
constexpr int kSmallMaxL = 512;
constexpr uint32_t kSmallChunk = 128 * 64 * 2;                       // 16 KB
// X (8 chunks), A and B (2 each), a 32 KB staging area (with A and B the
// three 32 KB slots of the prologue's bulk-copy ring), control words
constexpr uint32_t kSmallSmem = (kSmallMaxL / 64 + 2 + 2 + 2) * kSmallChunk + 256 + 1024;

struct SmallMat {
  const float* g;
  float* buf;
  float* w;           // W (step) or O (orthogonalize), m x n
  int m, n, trans, vec;
  int lp;             // long side padded to 64
};

struct SmallArgs {
  int nmats, ns_steps, nesterov, has_buf, assign;
  int debug_flags;      // bit 0: the CTA-pair kernel issues no first product; the four-CTA kernel
                        // keeps back CTA 1's first partial for CTA 0
  float mu, eps, a, b, c, lr;
  int* status;
  unsigned long long wait_limit_ns;
  SmallMat mats[kMaxMats];
};

// smem byte offset of element (row r, col c) in a chunked 128B-swizzled buffer
__device__ __forceinline__ uint32_t chunk_off(uint32_t r, uint32_t c) {
  return (c >> 6) * kSmallChunk + r * 128u + ((((c & 63u) >> 3) ^ (r & 7u)) << 4) + (c & 7u) * 2u;
}

__global__ void __launch_bounds__(kSmallThreads, 1) ns_small_kernel(const __grid_constant__ SmallArgs p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* Xs = smem;                                        // 8 chunks
  uint8_t* As = Xs + (kSmallMaxL / 64) * kSmallChunk;        // 2 chunks
  uint8_t* Bs = As + 2 * kSmallChunk;                        // 2 chunks
  uint8_t* Ss = Bs + 2 * kSmallChunk;                        // 2 chunks of staging
  uint64_t* mma_bar = reinterpret_cast<uint64_t*>(Ss + 2 * kSmallChunk);
  uint64_t* pro_bar = mma_bar + 1;                           // 3: prologue ring slots
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(pro_bar + 3);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
  float* red = reinterpret_cast<float*>(abort_flag + 1);     // 4 warp partials

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const SmallMat& M = p.mats[blockIdx.x];
  const int lp = M.lp;

  if (tid == 0) {
    mbar_init(mma_bar, 1);
    for (int i = 0; i < 3; ++i) mbar_init(&pro_bar[i], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  griddep_launch_dependents();
  griddep_wait();
  WaitCtx wc{abort_flag, p.status, p.wait_limit_ns, 0u};

  // ---- momentum, norm, X0 (bf16) into shared memory; zero padding included.
  const float* __restrict__ gp = M.g;
  float* __restrict__ bp = M.buf;
  float ss = 0.f;
  bool ok = true;
  if (M.vec) {
    // One SM moves all of g and buf: they stream through shared memory by 1-D
    // bulk copies (no registers held, many bytes in flight) in pieces of whole
    // rows of at most 16 KB each, through three (g, buf) slots in A | B | S,
    // two pieces in flight ahead of the one being processed; the new buffer
    // goes back by bulk store from the same slot.
    const int kx = M.trans ? M.n : M.m, lx = M.trans ? M.m : M.n;   // X is kx x lx
    // zero the padding of X first (rows >= kx, columns >= lx)
    for (int u = tid; u < kSmallMaxK * (lp / 8); u += kSmallThreads) {
      const int r = u / (lp / 8), c0 = 8 * (u % (lp / 8));
      if (r >= kx || c0 + 8 > lx) *reinterpret_cast<uint4*>(Xs + chunk_off((uint32_t)r, (uint32_t)c0)) = make_uint4(0, 0, 0, 0);
    }
    uint8_t* slots = As;
    const int rows_per = max(1, min(M.m, 4096 / M.n));
    const int npieces = (M.m + rows_per - 1) / rows_per;
    auto issue = [&](int pc) {
      const int sl = pc % 3;
      const uint32_t bytes = (uint32_t)(min(rows_per, M.m - pc * rows_per) * M.n * 4);
      const size_t off = (size_t)pc * rows_per * M.n;
      mbar_arrive_expect_tx(&pro_bar[sl], p.has_buf ? 2 * bytes : bytes);
      bulk_load(slots + sl * 32768, gp + off, bytes, &pro_bar[sl]);
      if (p.has_buf) bulk_load(slots + sl * 32768 + 16384, bp + off, bytes, &pro_bar[sl]);
    };
    if (tid == 0) {
      issue(0);
      if (npieces > 1) issue(1);
    }
    __syncthreads();                                         // padding zeroed before X is written
    for (int pc = 0; pc < npieces; ++pc) {
      const int sl = pc % 3;
      ok = __syncthreads_and(ok && mbar_wait(&pro_bar[sl], (uint32_t)((pc / 3) & 1), wc, kDevTimeoutFull)) != 0;
      if (!ok) break;
      float* sg = reinterpret_cast<float*>(slots + sl * 32768);
      float* sb = reinterpret_cast<float*>(slots + sl * 32768 + 16384);
      const int row0 = pc * rows_per;
      const int nel = min(rows_per, M.m - row0) * M.n;
      for (int e = tid * 4; e < nel; e += kSmallThreads * 4) {
        const float4 g4 = *reinterpret_cast<const float4*>(sg + e);
        float4 b4 = make_float4(0.f, 0.f, 0.f, 0.f);
        if (p.has_buf) b4 = *reinterpret_cast<const float4*>(sb + e);
        float gv[4] = {g4.x, g4.y, g4.z, g4.w}, bv[4] = {b4.x, b4.y, b4.z, b4.w}, G[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          G[q] = nesterov_g(gv[q], bv[q], p.mu, p.nesterov, p.has_buf);
          ss = fmaf(G[q], G[q], ss);
        }
        if (p.has_buf) *reinterpret_cast<float4*>(sb + e) = make_float4(bv[0], bv[1], bv[2], bv[3]);
        const int i = row0 + e / M.n, j = e % M.n;           // G row i, columns j..j+3
        if (!M.trans) {
          *reinterpret_cast<uint2*>(Xs + chunk_off((uint32_t)i, (uint32_t)j)) =
              make_uint2(pack_bf16x2(G[0], G[1]), pack_bf16x2(G[2], G[3]));
        } else {
#pragma unroll
          for (int q = 0; q < 4; ++q)
            *reinterpret_cast<__nv_bfloat16*>(Xs + chunk_off((uint32_t)(j + q), (uint32_t)i)) =
                __float2bfloat16_rn(G[q]);
        }
      }
      if (p.has_buf) fence_async_shared();                   // the new buffer values -> the bulk store
      __syncthreads();
      if (tid == 0) {
        if (p.has_buf) {
          bulk_store(bp + (size_t)row0 * M.n, sb, (uint32_t)(nel * 4));
          tma_store_commit();
        }
        if (pc + 2 < npieces) {
          tma_store_wait_read1();                            // slot (pc + 2) % 3 was stored from last time
          issue(pc + 2);
        }
      }
    }
    if (tid == 0) tma_store_wait_all0();                     // buf written; slots free for A and B
  } else {
  // Rows not 16-byte aligned: plain loads.  Each thread issues all loads of a
  // batch before any store (one CTA per SM has few warps to hide latency with).
  auto load4 = [&](size_t off, int col, int ncols, float (&gv)[4], float (&bv)[4]) {
    if (M.vec && col + 3 < ncols) {
      const float4 g4 = __ldg(reinterpret_cast<const float4*>(gp + off));
      gv[0] = g4.x; gv[1] = g4.y; gv[2] = g4.z; gv[3] = g4.w;
      if (p.has_buf) {
        const float4 b4 = *reinterpret_cast<const float4*>(bp + off);
        bv[0] = b4.x; bv[1] = b4.y; bv[2] = b4.z; bv[3] = b4.w;
      }
    } else {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        if (col + q < ncols) {
          gv[q] = gp[off + q];
          if (p.has_buf) bv[q] = bp[off + q];
        }
      }
    }
  };
  auto store4 = [&](size_t off, int col, int ncols, const float (&bv)[4]) {
    if (!p.has_buf) return;
    if (M.vec && col + 3 < ncols) {
      *reinterpret_cast<float4*>(bp + off) = make_float4(bv[0], bv[1], bv[2], bv[3]);
    } else {
#pragma unroll
      for (int q = 0; q < 4; ++q)
        if (col + q < ncols) bp[off + q] = bv[q];
    }
  };
  if (!M.trans) {
    // X[i][j] = G[i][j]: a batch is 2 rows x up to 4 steps of 128 columns
    for (int i0 = warp; i0 < kSmallMaxK; i0 += 8) {
      float gv[2][4][4], bv[2][4][4];
#pragma unroll
      for (int rr = 0; rr < 2; ++rr)
#pragma unroll
        for (int cs = 0; cs < 4; ++cs) {
#pragma unroll
          for (int q = 0; q < 4; ++q) { gv[rr][cs][q] = 0.f; bv[rr][cs][q] = 0.f; }
          const int i = i0 + 4 * rr, j = cs * 128 + 4 * lane;
          if (i < M.m && j < M.n) load4((size_t)i * M.n + j, j, M.n, gv[rr][cs], bv[rr][cs]);
        }
#pragma unroll
      for (int rr = 0; rr < 2; ++rr)
#pragma unroll
        for (int cs = 0; cs < 4; ++cs) {
          const int i = i0 + 4 * rr, j = cs * 128 + 4 * lane;
          if (j >= lp) continue;
          float G[4] = {0.f, 0.f, 0.f, 0.f};
          if (i < M.m && j < M.n) {
#pragma unroll
            for (int q = 0; q < 4; ++q)
              if (j + q < M.n) G[q] = nesterov_g(gv[rr][cs][q], bv[rr][cs][q], p.mu, p.nesterov, p.has_buf);
            store4((size_t)i * M.n + j, j, M.n, bv[rr][cs]);
          }
#pragma unroll
          for (int q = 0; q < 4; ++q) ss = fmaf(G[q], G[q], ss);
          *reinterpret_cast<uint2*>(Xs + chunk_off((uint32_t)i, (uint32_t)j)) =
              make_uint2(pack_bf16x2(G[0], G[1]), pack_bf16x2(G[2], G[3]));
        }
    }
  } else {
    // X[j][i] = G[i][j]: a warp reads rows i of G (n <= 128 columns), 8 rows per batch
    for (int i0 = warp; i0 < lp; i0 += 32) {
      float gv[8][4], bv[8][4];
      const int j = 4 * lane;                                 // X rows j..j+3
#pragma unroll
      for (int t = 0; t < 8; ++t) {
#pragma unroll
        for (int q = 0; q < 4; ++q) { gv[t][q] = 0.f; bv[t][q] = 0.f; }
        const int i = i0 + 4 * t;
        if (i < M.m && j < M.n) load4((size_t)i * M.n + j, j, M.n, gv[t], bv[t]);
      }
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        const int i = i0 + 4 * t;
        if (i >= lp) continue;
        float G[4] = {0.f, 0.f, 0.f, 0.f};
        if (i < M.m && j < M.n) {
#pragma unroll
          for (int q = 0; q < 4; ++q)
            if (j + q < M.n) G[q] = nesterov_g(gv[t][q], bv[t][q], p.mu, p.nesterov, p.has_buf);
          store4((size_t)i * M.n + j, j, M.n, bv[t]);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          ss = fmaf(G[q], G[q], ss);
          *reinterpret_cast<__nv_bfloat16*>(Xs + chunk_off((uint32_t)(j + q), (uint32_t)i)) =
              __float2bfloat16_rn(G[q]);
        }
      }
    }
  }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if (lane == 0) red[warp] = ss;
  fence_async_shared();                                      // X0 visible to the tensor core
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const float scale = 1.0f / ((float)sqrt((double)red[0] + (double)red[1] + (double)red[2] + (double)red[3]) + p.eps);
  const uint32_t tmem = *tmem_slot;
  const uint32_t tl = tmem + ((uint32_t)(warp * 32) << 16);  // this warp's 32 lanes
  const int r = warp * 32 + lane;                            // row of X / A / B owned by this thread
  uint32_t phase = 0;

  auto wait_mma = [&]() {
    bool got = ok && mbar_wait(mma_bar, phase, wc, kDevTimeoutAccum);
    phase ^= 1u;
    ok = __syncthreads_and(got) != 0;
    tc_fence_after();
  };
  auto publish_smem = [&]() {                                // generic writes -> next MMAs
    fence_async_shared();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  };

  // W -= lr * O (or O = result) for X columns cc*32 .. +31 of this thread's row
  // r: staged in the A buffer (free at that point), then read-modified-written
  // in whole 128-byte rows with all loads of a thread in flight at once
  auto apply_chunk = [&](int cc, const float* v) {
        float* S = reinterpret_cast<float*>(As);
        if (!M.trans) {
#pragma unroll
          for (int j = 0; j < 8; ++j)
            *reinterpret_cast<float4*>(S + r * 32 + ((j ^ (r & 7)) << 2)) =
                make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
        } else {
#pragma unroll
          for (int q = 0; q < 32; ++q) S[q * 128 + r] = v[q];
        }
        __syncthreads();
        float4 o[8], w4[8];
        float* wp[8];
        bool okw[8], full[8];
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          const int idx = tid + kSmallThreads * t;
          int wi, wj;
          if (!M.trans) {
            const int row = idx >> 3, qd = idx & 7;
            wi = row; wj = cc * 32 + 4 * qd;
            o[t] = *reinterpret_cast<const float4*>(S + row * 32 + ((qd ^ (row & 7)) << 2));
          } else {
            const int c = idx >> 5, qd = idx & 31;
            wi = cc * 32 + c; wj = 4 * qd;
            o[t] = *reinterpret_cast<const float4*>(S + c * 128 + 4 * qd);
          }
          okw[t] = wi < M.m && wj < M.n;
          full[t] = M.vec && wj + 3 < M.n;
          wp[t] = M.w + (size_t)wi * M.n + wj;
          w4[t] = make_float4(0.f, 0.f, 0.f, 0.f);
          if (okw[t] && full[t] && !p.assign) w4[t] = *reinterpret_cast<const float4*>(wp[t]);
        }
#pragma unroll
        for (int t = 0; t < 8; ++t) {
          if (!okw[t]) continue;
          if (full[t]) {
            float4 r4 = w4[t];
            if (p.assign) r4 = o[t];
            else { r4.x -= p.lr * o[t].x; r4.y -= p.lr * o[t].y; r4.z -= p.lr * o[t].z; r4.w -= p.lr * o[t].w; }
            *reinterpret_cast<float4*>(wp[t]) = r4;
          } else {
            const float ov[4] = {o[t].x, o[t].y, o[t].z, o[t].w};
            const int wj = (int)((wp[t] - M.w) % M.n);
            for (int e = 0; e < 4 && wj + e < M.n; ++e) wp[t][e] = p.assign ? ov[e] : wp[t][e] - p.lr * ov[e];
          }
        }
        __syncthreads();
  };

  for (int it = 0; it < p.ns_steps && ok; ++it) {
    const float s = it == 0 ? scale : 1.0f;
    const bool last = it == p.ns_steps - 1;
    // A = s^2 X X^T : M = N = 128, K = lp
    if (tid == 0) {
      const uint32_t idesc = idesc_bf16_f32(128, 128, 0, 0);
      for (int kk = 0; kk < lp / 16; ++kk) {
        const uint32_t a = smem_u32(Xs) + (kk >> 2) * kSmallChunk + (kk & 3) * 32;
        const uint64_t d = smem_desc_sw128(a, 16, 1024);
        tc_mma_bf16(tmem, d, d, idesc, kk > 0 ? 1u : 0u);
      }
      tc_commit(mma_bar);
    }
    wait_mma();
    if (!ok) break;
#pragma unroll 1
    for (int c64 = 0; c64 < 2; ++c64) {
      float v[64];
      tmem_ld_32x32b_x64(tl + (uint32_t)(c64 * 64), v);
#pragma unroll
      for (int q = 0; q < 64; q += 8) {
        uint4 o;
        o.x = pack_bf16x2(s * s * v[q], s * s * v[q + 1]);
        o.y = pack_bf16x2(s * s * v[q + 2], s * s * v[q + 3]);
        o.z = pack_bf16x2(s * s * v[q + 4], s * s * v[q + 5]);
        o.w = pack_bf16x2(s * s * v[q + 6], s * s * v[q + 7]);
        *reinterpret_cast<uint4*>(As + chunk_off((uint32_t)r, (uint32_t)(c64 * 64 + q))) = o;
      }
    }
    publish_smem();
    // B = b A + c A A : M = N = K = 128 (A symmetric: both operands K-major rows of A)
    if (tid == 0) {
      const uint32_t idesc = idesc_bf16_f32(128, 128, 0, 0);
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t a = smem_u32(As) + (kk >> 2) * kSmallChunk + (kk & 3) * 32;
        const uint64_t d = smem_desc_sw128(a, 16, 1024);
        tc_mma_bf16(tmem, d, d, idesc, kk > 0 ? 1u : 0u);
      }
      tc_commit(mma_bar);
    }
    wait_mma();
    if (!ok) break;
#pragma unroll 1
    for (int c64 = 0; c64 < 2; ++c64) {
      float v[64];
      tmem_ld_32x32b_x64(tl + (uint32_t)(c64 * 64), v);
#pragma unroll
      for (int q = 0; q < 64; q += 8) {
        const uint4 araw = *reinterpret_cast<const uint4*>(As + chunk_off((uint32_t)r, (uint32_t)(c64 * 64 + q)));
        const __nv_bfloat162* ah = reinterpret_cast<const __nv_bfloat162*>(&araw);
        float o8[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(ah[e]);
          o8[2 * e] = fmaf(p.c, v[q + 2 * e], p.b * f.x);
          o8[2 * e + 1] = fmaf(p.c, v[q + 2 * e + 1], p.b * f.y);
        }
        *reinterpret_cast<uint4*>(Bs + chunk_off((uint32_t)r, (uint32_t)(c64 * 64 + q))) =
            make_uint4(pack_bf16x2(o8[0], o8[1]), pack_bf16x2(o8[2], o8[3]), pack_bf16x2(o8[4], o8[5]),
                       pack_bf16x2(o8[6], o8[7]));
      }
    }
    publish_smem();
    // X' = a s X + s B X : M = 128, N = lp (<= 256 per instruction), K = 128; X read MN-major
    if (tid == 0) {
      for (int n0 = 0; n0 < lp; n0 += 256) {
        const int nn = min(256, lp - n0);
        const uint32_t idesc = idesc_bf16_f32(128, (uint32_t)nn, 0, 1);
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t a = smem_u32(Bs) + (kk >> 2) * kSmallChunk + (kk & 3) * 32;
          const uint32_t b = smem_u32(Xs) + (n0 >> 6) * kSmallChunk + kk * (16 * 128);
          tc_mma_bf16(tmem + (uint32_t)n0, smem_desc_sw128(a, 16, 1024), smem_desc_sw128(b, kSmallChunk, 1024),
                      idesc, kk > 0 ? 1u : 0u);
        }
      }
      tc_commit(mma_bar);
    }
    wait_mma();
    if (!ok) break;
#pragma unroll 1
    for (int c64 = 0; c64 < lp / 64; ++c64) {
     float v64[64];
     tmem_ld_32x32b_x64(tl + (uint32_t)(c64 * 64), v64);
#pragma unroll
     for (int half = 0; half < 2; ++half) {
      const int cc = 2 * c64 + half;
      float* v = v64 + 32 * half;
#pragma unroll
      for (int q = 0; q < 32; q += 8) {
        const uint32_t xo = chunk_off((uint32_t)r, (uint32_t)(cc * 32 + q));
        const uint4 xraw = *reinterpret_cast<const uint4*>(Xs + xo);
        const __nv_bfloat162* xh = reinterpret_cast<const __nv_bfloat162*>(&xraw);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(xh[e]);
          v[q + 2 * e] = fmaf(s, v[q + 2 * e], p.a * s * f.x);
          v[q + 2 * e + 1] = fmaf(s, v[q + 2 * e + 1], p.a * s * f.y);
        }
        if (!last)
          *reinterpret_cast<uint4*>(Xs + xo) =
              make_uint4(pack_bf16x2(v[q], v[q + 1]), pack_bf16x2(v[q + 2], v[q + 3]),
                         pack_bf16x2(v[q + 4], v[q + 5]), pack_bf16x2(v[q + 6], v[q + 7]));
      }
      if (last) apply_chunk(cc, v);
     }
    }
    if (!last) publish_smem();
  }
  if (p.ns_steps == 0 && ok) {
    // O = s * X0 (the listing with an empty loop)
#pragma unroll 1
    for (int cc = 0; cc < lp / 32; ++cc) {
      float v[32];
#pragma unroll
      for (int q = 0; q < 32; q += 8) {
        const uint4 xraw = *reinterpret_cast<const uint4*>(Xs + chunk_off((uint32_t)r, (uint32_t)(cc * 32 + q)));
        const __nv_bfloat162* xh = reinterpret_cast<const __nv_bfloat162*>(&xraw);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(xh[e]);
          v[q + 2 * e] = scale * f.x;
          v[q + 2 * e + 1] = scale * f.y;
        }
      }
      apply_chunk(cc, v);
    }
  }
  tma_store_wait_all0();                                     // this thread's bulk copies are done
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ======================================== CTA-pair fused step, k <= 256 ===
// The whole step of a matrix with short side 128 < k <= 256 and long side
// l <= 256 on one cluster of two CTAs.  CTA r holds rows [128r, 128r + 128) of
// X (XO, all 256 columns), of A and then B' (AB), and all 256 rows of its own
// column half of X (XC: the update's N operand).  Every product is one
// tcgen05.mma.cta_group::2 with M = N = 256 issued by CTA 0:
//   Gram     A = s^2 X X^T         both operands XO (K-major, K = 256)
//   poly     B' = aI + bA + cAA     both operands AB (A symmetric)
//   update   X' = s B' X            AB (K-major) x XC (MN-major, K = X rows)
// and each CTA's TMEM holds its 128 rows x 256 fp32 columns.  The update's
// epilogue writes the peer's column half of its rows into the peer's XC
// through distributed shared memory.  Phases are separated by cluster
// barriers; both CTAs take every barrier on every path (a CTA whose bounded
// wait gave up only stops issuing and waiting), so neither can be left behind.
constexpr int kPairMaxK = 256;
constexpr int kPairMaxL = 256;
constexpr int kPairWarps = 8;        // two warpgroups: one per column half of the accumulator
constexpr int kPairThreads = 32 * kPairWarps;
constexpr uint32_t kPairXC = 256 * 64 * 2;                                   // 32 KB: 64 columns of 256 rows
constexpr uint32_t kPairSmem = 4 * kSmallChunk + 2 * kPairXC + 4 * kSmallChunk + 256 + 1024;

// Byte offset of element (row, c) in XC: 64-column chunks of 256 rows, 128-byte swizzle.
__device__ __forceinline__ uint32_t xc_off(uint32_t row, uint32_t c) {
  return (c >> 6) * kPairXC + row * 128u + ((((c & 63u) >> 3) ^ (row & 7u)) << 4) + (c & 7u) * 2u;
}

__global__ void __launch_bounds__(kPairThreads, 1) ns_pair_kernel(const __grid_constant__ SmallArgs p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* XO = smem;                                        // 4 chunks [128][64]
  uint8_t* XC = XO + 4 * kSmallChunk;                        // 2 chunks [256][64]
  uint8_t* AB = XC + 2 * kPairXC;                            // 4 chunks [128][64]
  uint64_t* mma_bar = reinterpret_cast<uint64_t*>(AB + 4 * kSmallChunk);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_bar + 1);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
  float* red = reinterpret_cast<float*>(abort_flag + 1);     // [0..7] warp partials, [8..9] CTA partials

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_ctarank(), peer = rank ^ 1u;
  const SmallMat& M = p.mats[cluster_id_x()];
  const int row_base = (int)rank * 128;                      // X rows of this CTA
  const uint32_t xc_peer = mapa_shared(XC, peer);            // the peer's XC (same layout)

  if (tid == 0) {
    mbar_init(mma_bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc_pair(tmem_slot, 256);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  griddep_launch_dependents();
  griddep_wait();
  // Stores one bf16 quad / element of X row `xr` (global), column j into XO
  // (local row) and into the XC of the CTA that owns column j's half.
  auto put_quad = [&](int xr, int j, uint32_t lo, uint32_t hi) {
    *reinterpret_cast<uint2*>(XO + chunk_off((uint32_t)(xr - row_base), (uint32_t)j)) = make_uint2(lo, hi);
    const uint32_t off = xc_off((uint32_t)xr, (uint32_t)(j & 127));
    if ((j >> 7) == (int)rank) *reinterpret_cast<uint2*>(XC + off) = make_uint2(lo, hi);
    else st_cluster_v2(xc_peer + off, lo, hi);
  };
  auto put_one = [&](int xr, int j, __nv_bfloat16 v) {
    *reinterpret_cast<__nv_bfloat16*>(XO + chunk_off((uint32_t)(xr - row_base), (uint32_t)j)) = v;
    const uint32_t off = xc_off((uint32_t)xr, (uint32_t)(j & 127));
    if ((j >> 7) == (int)rank) *reinterpret_cast<__nv_bfloat16*>(XC + off) = v;
    else st_cluster_u16(xc_peer + off, __bfloat16_as_ushort(v));
  };

  // ---- momentum, norm partial, X0 (bf16; zero padding included)
  const float* __restrict__ gp = M.g;
  float* __restrict__ bp = M.buf;
  float ss = 0.f;
  auto load4 = [&](size_t off, int col, int ncols, float (&gv)[4], float (&bv)[4]) {
    if (M.vec && col + 3 < ncols) {
      const float4 g4 = __ldg(reinterpret_cast<const float4*>(gp + off));
      gv[0] = g4.x; gv[1] = g4.y; gv[2] = g4.z; gv[3] = g4.w;
      if (p.has_buf) {
        const float4 b4 = *reinterpret_cast<const float4*>(bp + off);
        bv[0] = b4.x; bv[1] = b4.y; bv[2] = b4.z; bv[3] = b4.w;
      }
    } else {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        if (col + q < ncols) {
          gv[q] = gp[off + q];
          if (p.has_buf) bv[q] = bp[off + q];
        }
      }
    }
  };
  auto store4 = [&](size_t off, int col, int ncols, const float (&bv)[4]) {
    if (!p.has_buf) return;
    if (M.vec && col + 3 < ncols) {
      *reinterpret_cast<float4*>(bp + off) = make_float4(bv[0], bv[1], bv[2], bv[3]);
    } else {
#pragma unroll
      for (int q = 0; q < 4; ++q)
        if (col + q < ncols) bp[off + q] = bv[q];
    }
  };
  if (!M.trans) {
    // X row i = G row i: a batch is rows i0 and i0 + 8, 2 steps of 128 columns each
    for (int i0 = warp; i0 < 128; i0 += 2 * kPairWarps) {
      float gv[2][2][4], bv[2][2][4];
#pragma unroll
      for (int rr = 0; rr < 2; ++rr)
#pragma unroll
        for (int cs = 0; cs < 2; ++cs) {
#pragma unroll
          for (int q = 0; q < 4; ++q) { gv[rr][cs][q] = 0.f; bv[rr][cs][q] = 0.f; }
          const int i = row_base + i0 + kPairWarps * rr, j = cs * 128 + 4 * lane;
          if (i < M.m && j < M.n) load4((size_t)i * M.n + j, j, M.n, gv[rr][cs], bv[rr][cs]);
        }
#pragma unroll
      for (int rr = 0; rr < 2; ++rr)
#pragma unroll
        for (int cs = 0; cs < 2; ++cs) {
          const int i = row_base + i0 + kPairWarps * rr, j = cs * 128 + 4 * lane;
          float G[4] = {0.f, 0.f, 0.f, 0.f};
          if (i < M.m && j < M.n) {
#pragma unroll
            for (int q = 0; q < 4; ++q)
              if (j + q < M.n) G[q] = nesterov_g(gv[rr][cs][q], bv[rr][cs][q], p.mu, p.nesterov, p.has_buf);
            store4((size_t)i * M.n + j, j, M.n, bv[rr][cs]);
          }
#pragma unroll
          for (int q = 0; q < 4; ++q) ss = fmaf(G[q], G[q], ss);
          put_quad(i, j, pack_bf16x2(G[0], G[1]), pack_bf16x2(G[2], G[3]));
        }
    }
  } else {
    // X row j = G column j (this CTA's 128 columns of G), X column i = G row i;
    // a batch is 8 rows of G, kPairWarps apart
    for (int i0 = warp; i0 < kPairMaxL; i0 += 8 * kPairWarps) {
      float gv[8][4], bv[8][4];
      const int j = row_base + 4 * lane;                      // X rows j..j+3
#pragma unroll
      for (int t = 0; t < 8; ++t) {
#pragma unroll
        for (int q = 0; q < 4; ++q) { gv[t][q] = 0.f; bv[t][q] = 0.f; }
        const int i = i0 + kPairWarps * t;
        if (i < M.m && j < M.n) load4((size_t)i * M.n + j, j, M.n, gv[t], bv[t]);
      }
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        const int i = i0 + kPairWarps * t;
        float G[4] = {0.f, 0.f, 0.f, 0.f};
        if (i < M.m && j < M.n) {
#pragma unroll
          for (int q = 0; q < 4; ++q)
            if (j + q < M.n) G[q] = nesterov_g(gv[t][q], bv[t][q], p.mu, p.nesterov, p.has_buf);
          store4((size_t)i * M.n + j, j, M.n, bv[t]);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          ss = fmaf(G[q], G[q], ss);
          put_one(j + q, i, __float2bfloat16_rn(G[q]));
        }
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if (lane == 0) red[warp] = ss;
  __syncthreads();
  if (tid == 0) {
    float part = 0.f;
    for (int w = 0; w < kPairWarps; ++w) part += red[w];
    red[kPairWarps + rank] = part;
    st_cluster_u32(mapa_shared(&red[kPairWarps + rank], peer), __float_as_uint(part));
  }
  fence_async_all();                                         // X0 (local and peer writes) -> tensor core
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  const float scale =
      1.0f / ((float)sqrt((double)red[kPairWarps] + (double)red[kPairWarps + 1]) + p.eps);
  const uint32_t tmem = *tmem_slot;
  const int q4 = warp & 3;                                   // TMEM lane quarter of this warp
  const int hw = warp >> 2;                                  // column half of the accumulator it reads
  const uint32_t tl = tmem + ((uint32_t)(q4 * 32) << 16);    // this warp's 32 lanes
  const int r = q4 * 32 + lane;                              // local row owned by this thread
  const bool leader = rank == 0 && tid == 0;
  WaitCtx wc{abort_flag, p.status, p.wait_limit_ns, mapa_shared(abort_flag, peer)};
  bool ok = true;
  uint32_t phase = 0;

  auto commit_both = [&]() {
    tc_commit_pair(mapa_shared(mma_bar, 0));
    tc_commit_pair(mapa_shared(mma_bar, 1));
  };
  auto wait_mma = [&]() {
    bool got = ok && mbar_wait(mma_bar, phase, wc, kDevTimeoutAccum);
    phase ^= 1u;
    ok = __syncthreads_and(got) != 0;
    tc_fence_after();
  };
  auto publish = [&]() {                                     // this phase's writes -> the next MMAs
    fence_async_all();
    tc_fence_before();
    cluster_sync_all();
    tc_fence_after();
  };
  // One apply round: every thread holds 32 values of its row, X columns
  // 128 hw + 32 j .. +31; the two halves stage theirs in AB (free once the
  // update's MMAs are done) and all threads write both chunks to W (or O)
  // in whole 128-byte rows.
  auto apply_round = [&](int j, const float* v) {
    float* Sh = reinterpret_cast<float*>(AB + hw * 16384);
    if (!M.trans) {
#pragma unroll
      for (int u = 0; u < 8; ++u)
        *reinterpret_cast<float4*>(Sh + r * 32 + ((u ^ (r & 7)) << 2)) =
            make_float4(v[4 * u], v[4 * u + 1], v[4 * u + 2], v[4 * u + 3]);
    } else {
#pragma unroll
      for (int c = 0; c < 32; ++c) Sh[c * 128 + r] = v[c];
    }
    __syncthreads();
    float4 o[8], w4[8];
    float* wp[8];
    bool okw[8], full[8];
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      const int idx = tid + kPairThreads * t;               // 2 staged chunks x 1024 float4
      const int sel = idx >> 10, loc = idx & 1023;
      const int cc = 4 * sel + j;                            // 32-column chunk of X
      const float* S = reinterpret_cast<const float*>(AB + sel * 16384);
      int wi, wj;
      if (!M.trans) {
        const int row = loc >> 3, qd = loc & 7;
        wi = row_base + row; wj = cc * 32 + 4 * qd;
        o[t] = *reinterpret_cast<const float4*>(S + row * 32 + ((qd ^ (row & 7)) << 2));
      } else {
        const int c = loc >> 5, qd = loc & 31;
        wi = cc * 32 + c; wj = row_base + 4 * qd;
        o[t] = *reinterpret_cast<const float4*>(S + c * 128 + 4 * qd);
      }
      okw[t] = wi < M.m && wj < M.n;
      full[t] = M.vec && wj + 3 < M.n;
      wp[t] = M.w + (size_t)wi * M.n + wj;
      w4[t] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (okw[t] && full[t] && !p.assign) w4[t] = *reinterpret_cast<const float4*>(wp[t]);
    }
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      if (!okw[t]) continue;
      if (full[t]) {
        float4 r4 = w4[t];
        if (p.assign) r4 = o[t];
        else { r4.x -= p.lr * o[t].x; r4.y -= p.lr * o[t].y; r4.z -= p.lr * o[t].z; r4.w -= p.lr * o[t].w; }
        *reinterpret_cast<float4*>(wp[t]) = r4;
      } else {
        const float ov[4] = {o[t].x, o[t].y, o[t].z, o[t].w};
        const int wj = (int)((wp[t] - M.w) % M.n);
        for (int e = 0; e < 4 && wj + e < M.n; ++e) wp[t][e] = p.assign ? ov[e] : wp[t][e] - p.lr * ov[e];
      }
    }
    __syncthreads();
  };

  const uint32_t idesc_kk = idesc_bf16_f32(256, 256, 0, 0);
  for (int it = 0; it < p.ns_steps; ++it) {
    const float s = it == 0 ? scale : 1.0f;
    const bool last = it == p.ns_steps - 1;
    // ---- Gram: A = s^2 X X^T
    const bool inject_skip = (p.debug_flags & 1) && it == 0;
    if (leader && ok && !inject_skip) {
      for (int kk = 0; kk < 16; ++kk) {
        const uint64_t d = smem_desc_sw128(smem_u32(XO) + (kk >> 2) * kSmallChunk + (kk & 3) * 32, 16, 1024);
        tc_mma_bf16_pair(tmem, d, d, idesc_kk, kk > 0 ? 1u : 0u);
      }
      commit_both();
    }
    wait_mma();
#pragma unroll 1
    for (int jj = 0; jj < 2 && ok; ++jj) {
      const int c64 = 2 * hw + jj;
      float v[64];
      tmem_ld_32x32b_x64(tl + (uint32_t)(c64 * 64), v);
#pragma unroll
      for (int q = 0; q < 64; q += 8) {
        uint4 o;
        o.x = pack_bf16x2(s * s * v[q], s * s * v[q + 1]);
        o.y = pack_bf16x2(s * s * v[q + 2], s * s * v[q + 3]);
        o.z = pack_bf16x2(s * s * v[q + 4], s * s * v[q + 5]);
        o.w = pack_bf16x2(s * s * v[q + 6], s * s * v[q + 7]);
        *reinterpret_cast<uint4*>(AB + chunk_off((uint32_t)r, (uint32_t)(c64 * 64 + q))) = o;
      }
    }
    publish();
    // ---- polynomial: B' = aI + bA + cAA, in place over A
    if (leader && ok) {
      for (int kk = 0; kk < 16; ++kk) {
        const uint64_t d = smem_desc_sw128(smem_u32(AB) + (kk >> 2) * kSmallChunk + (kk & 3) * 32, 16, 1024);
        tc_mma_bf16_pair(tmem, d, d, idesc_kk, kk > 0 ? 1u : 0u);
      }
      commit_both();
    }
    wait_mma();
    const int dcol = row_base + r;                           // this row's diagonal column
#pragma unroll 1
    for (int jj = 0; jj < 2 && ok; ++jj) {
      const int c64 = 2 * hw + jj;
      float v[64];
      tmem_ld_32x32b_x64(tl + (uint32_t)(c64 * 64), v);
#pragma unroll
      for (int q = 0; q < 64; q += 8) {
        uint8_t* ap = AB + chunk_off((uint32_t)r, (uint32_t)(c64 * 64 + q));
        const uint4 araw = *reinterpret_cast<const uint4*>(ap);
        const __nv_bfloat162* ah = reinterpret_cast<const __nv_bfloat162*>(&araw);
        float o8[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(ah[e]);
          const int c0 = c64 * 64 + q + 2 * e;
          o8[2 * e] = fmaf(p.c, v[q + 2 * e], p.b * f.x) + (c0 == dcol ? p.a : 0.f);
          o8[2 * e + 1] = fmaf(p.c, v[q + 2 * e + 1], p.b * f.y) + (c0 + 1 == dcol ? p.a : 0.f);
        }
        *reinterpret_cast<uint4*>(ap) = make_uint4(pack_bf16x2(o8[0], o8[1]), pack_bf16x2(o8[2], o8[3]),
                                                   pack_bf16x2(o8[4], o8[5]), pack_bf16x2(o8[6], o8[7]));
      }
    }
    publish();
    // ---- update: X' = s B' X (X read MN-major from XC: K = the 256 rows of X)
    if (leader && ok) {
      const uint32_t idesc = idesc_bf16_f32(256, 256, 0, 1);
      for (int kk = 0; kk < 16; ++kk) {
        const uint64_t a = smem_desc_sw128(smem_u32(AB) + (kk >> 2) * kSmallChunk + (kk & 3) * 32, 16, 1024);
        const uint64_t b = smem_desc_sw128(smem_u32(XC) + kk * (16 * 128), kPairXC, 1024);
        tc_mma_bf16_pair(tmem, a, b, idesc, kk > 0 ? 1u : 0u);
      }
      commit_both();
    }
    wait_mma();
#pragma unroll 1
    for (int jj = 0; jj < 2 && ok; ++jj) {
      const int c64 = 2 * hw + jj;
      float v[64];
      tmem_ld_32x32b_x64(tl + (uint32_t)(c64 * 64), v);
#pragma unroll
      for (int i = 0; i < 64; ++i) v[i] *= s;
      if (last) {
        apply_round(2 * jj, v);
        apply_round(2 * jj + 1, v + 32);
      } else {
#pragma unroll
        for (int q = 0; q < 64; q += 8) {
          const int j = c64 * 64 + q;
          const uint4 o = make_uint4(pack_bf16x2(v[q], v[q + 1]), pack_bf16x2(v[q + 2], v[q + 3]),
                                     pack_bf16x2(v[q + 4], v[q + 5]), pack_bf16x2(v[q + 6], v[q + 7]));
          *reinterpret_cast<uint4*>(XO + chunk_off((uint32_t)r, (uint32_t)j)) = o;
          const uint32_t off = xc_off((uint32_t)(row_base + r), (uint32_t)(j & 127));
          if ((j >> 7) == (int)rank) *reinterpret_cast<uint4*>(XC + off) = o;
          else st_cluster_v4(xc_peer + off, o);
        }
      }
    }
    if (!last) publish();
  }
  if (p.ns_steps == 0 && ok) {
    // O = s * X0 (the listing with an empty loop)
#pragma unroll 1
    for (int j = 0; j < 4; ++j) {
      const int cc = 4 * hw + j;
      float v[32];
#pragma unroll
      for (int q = 0; q < 32; q += 8) {
        const uint4 xraw = *reinterpret_cast<const uint4*>(XO + chunk_off((uint32_t)r, (uint32_t)(cc * 32 + q)));
        const __nv_bfloat162* xh = reinterpret_cast<const __nv_bfloat162*>(&xraw);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(xh[e]);
          v[q + 2 * e] = scale * f.x;
          v[q + 2 * e + 1] = scale * f.y;
        }
      }
      apply_round(j, v);
    }
  }
  tc_fence_before();
  cluster_sync_all();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 256);
  }
}

// ============================================= small matrices, four CTAs ===
// The whole step of one small matrix (short side k <= 128, long side
// 256 < l <= 512) on a cluster of four CTAs, each holding 128 columns of X (a
// quarter of the long side), so that the memory phases (g, buf and W) and the
// quarter-sized products run on four SMs instead of one.  The Gram matrix is a
// sum over the quarters: every CTA computes its partial X_q X_q^T in TMEM, and
// warp r stages row block r of it (32 rows, fp32) in shared memory and sends it
// by one bulk copy into CTA r's inbox, counted on an mbarrier there; CTA r
// adds the four partials of its rows in a fixed order and sends those rows of
// A (bf16) by bulk copies into every other CTA, counted on a second mbarrier.
// Each CTA then forms the whole polynomial matrix B = b A + c A A (128 x 128,
// from its own copy of A) and the update of its own quarter,
// X_q' = a s X_q + s B X_q.  No cluster barrier separates the iterations:
// every copy into a buffer follows, through this chain of waits, the
// receiver's last read of it (a partial of iteration i+1 is sent only after
// its sender received every A row of iteration i, which each owner sends only
// after summing its inbox; A rows of i+1 leave their owner only after every
// CTA's partial of i+1, sent after that CTA's last read of A of iteration i).
// Waits are bounded; a CTA that gave up stops sending and waiting, and the
// cluster barriers at the start and the end are taken on every path.
// 16-byte asynchronous copy global -> shared memory (bypassing L1) and the
// wait for all of this thread's copies.
__device__ __forceinline__ void cp_async_16(void* smem_dst, const void* gsrc) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)), "l"(gsrc) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
// Bulk copy of `bytes` (a multiple of 16, both addresses 16-byte aligned) from
// this CTA's shared memory into a CTA of the cluster; the bytes are counted on
// an mbarrier in the destination CTA (cluster addresses).
__device__ __forceinline__ void bulk_copy_to_cta(uint32_t dst_cluster, const void* src, uint32_t bytes,
                                                 uint32_t bar_cluster) {
  asm volatile("cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               ::"r"(dst_cluster), "r"(smem_u32(src)), "r"(bytes), "r"(bar_cluster)
               : "memory");
}

constexpr int kQuadThreads = 128;
constexpr int kQuadCols = 128;                 // columns of X held by one CTA
constexpr int kQuadMaxMats = 37;               // four CTAs each: one wave of 148 SMs
// [sender][row rr of this CTA's block][16-byte unit] fp32, unit u of row rr
// stored at (u + rr) mod 32 so that the 32 rows' writes and reads hit
// different banks
constexpr uint32_t kQuadSlot = 32 * 128 * 4;                 // one sender's 32 rows of a partial (fp32)
constexpr uint32_t kQuadInbox = 4 * kQuadSlot;
constexpr uint32_t kQuadOutbox = 3 * kQuadSlot;               // this CTA's rows for the other three CTAs
constexpr uint32_t kQuadARows = 32 * 64 * 2;                  // 32 rows of one 64-column chunk of A (bf16)
__device__ __forceinline__ uint32_t quad_inbox_off(uint32_t q, uint32_t rr, uint32_t u) {
  return ((q * 32u + rr) * 32u + ((u + rr) & 31u)) * 16u;
}
constexpr uint32_t kQuadSmem = 6 * kSmallChunk + kQuadInbox + kQuadOutbox + 256 + 1024;
static_assert(kQuadSmem <= 232448, "more dynamic shared memory than a CTA may have");

__global__ void __launch_bounds__(kQuadThreads, 1) ns_quad_kernel(const __grid_constant__ SmallArgs p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* Xs = smem;                                        // 2 chunks: this CTA's 128 columns of X
  uint8_t* As = Xs + 2 * kSmallChunk;                        // 2 chunks: A
  uint8_t* Bs = As + 2 * kSmallChunk;                        // 2 chunks: B
  float* inbox = reinterpret_cast<float*>(Bs + 2 * kSmallChunk);
  uint8_t* outbox = reinterpret_cast<uint8_t*>(inbox) + kQuadInbox;
  uint64_t* mma_bar = reinterpret_cast<uint64_t*>(outbox + kQuadOutbox);
  uint64_t* inbox_bar = mma_bar + 1;                         // the three other CTAs' partials of this CTA's rows
  uint64_t* a_bar = mma_bar + 2;                             // the three other CTAs' rows of A
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_bar + 3);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
  float* red = reinterpret_cast<float*>(abort_flag + 1);    // [0..3] warp partials, [4..7] the CTAs' partials

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_ctarank();
  const SmallMat& M = p.mats[cluster_id_x()];
  const int c0 = (int)rank * kQuadCols;                      // first X column of this CTA

  if (tid == 0) {
    mbar_init(mma_bar, 1);
    mbar_init(inbox_bar, 1);
    mbar_init(a_bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  cluster_sync_all();                                        // every CTA initialised before any remote write
  tc_fence_after();
  griddep_launch_dependents();
  griddep_wait();
  WaitCtx wc{abort_flag, p.status, p.wait_limit_ns, 0u};

  // ---- momentum, norm partial, this CTA's quarter of X0 (bf16, padding zero)
  const float* __restrict__ gp = M.g;
  float* __restrict__ bp = M.buf;
  auto load4 = [&](size_t off, int col, int ncols, float (&gv)[4], float (&bv)[4]) {
    if (M.vec && col + 3 < ncols) {
      const float4 g4 = __ldg(reinterpret_cast<const float4*>(gp + off));
      gv[0] = g4.x; gv[1] = g4.y; gv[2] = g4.z; gv[3] = g4.w;
      if (p.has_buf) {
        const float4 b4 = *reinterpret_cast<const float4*>(bp + off);
        bv[0] = b4.x; bv[1] = b4.y; bv[2] = b4.z; bv[3] = b4.w;
      }
    } else {
#pragma unroll
      for (int q = 0; q < 4; ++q)
        if (col + q < ncols) {
          gv[q] = gp[off + q];
          if (p.has_buf) bv[q] = bp[off + q];
        }
    }
  };
  auto store4 = [&](size_t off, int col, int ncols, const float (&bv)[4]) {
    if (!p.has_buf) return;
    if (M.vec && col + 3 < ncols) {
      *reinterpret_cast<float4*>(bp + off) = make_float4(bv[0], bv[1], bv[2], bv[3]);
    } else {
#pragma unroll
      for (int q = 0; q < 4; ++q)
        if (col + q < ncols) bp[off + q] = bv[q];
    }
  };
  float ss = 0.f;
  // Aligned rows: the CTA's 128 x 128 blocks of g and buf land in shared
  // memory by asynchronous copies, all in flight at once (g in the inbox,
  // buf in A | B, both free until the first product), then each warp walks
  // rows of them.  Otherwise: plain loads, eight rows per batch.
  const bool staged = M.vec;
  const int gr0 = M.trans ? c0 : 0, gc0 = M.trans ? 0 : c0;  // block origin in g: G rows, G columns
  float* Sg = inbox;
  float* Sb = reinterpret_cast<float*>(As);
  if (staged) {
    for (int e = tid; e < 128 * 32; e += kQuadThreads) {
      const int i = e >> 5, u = e & 31;                      // block row, 16-byte unit
      const int gi = gr0 + i, gj = gc0 + 4 * u;
      if (gi < M.m && gj < M.n) {
        const size_t off = (size_t)gi * M.n + gj;
        cp_async_16(Sg + i * 128 + 4 * u, gp + off);
        if (p.has_buf) cp_async_16(Sb + i * 128 + 4 * u, bp + off);
      }
    }
    cp_async_wait_all();
    __syncthreads();
  }
  // G[i][j] for G row i = i0 + 4 t (eight per batch, all loads first), G columns
  // j .. j+3 with j = jb + 4 lane
  auto batch = [&](int i0, int jb, auto&& put) {
    if (staged) {
      const int j = jb + 4 * lane;
#pragma unroll 2
      for (int t = 0; t < 8; ++t) {
        const int i = i0 + 4 * t;
        float G[4] = {0.f, 0.f, 0.f, 0.f};
        if (i < M.m && j < M.n) {
          const int so = (i - gr0) * 128 + (j - gc0);
          const float4 g4 = *reinterpret_cast<const float4*>(Sg + so);
          float4 b4 = make_float4(0.f, 0.f, 0.f, 0.f);
          if (p.has_buf) b4 = *reinterpret_cast<const float4*>(Sb + so);
          float gv[4] = {g4.x, g4.y, g4.z, g4.w}, bv[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
          for (int q = 0; q < 4; ++q) G[q] = nesterov_g(gv[q], bv[q], p.mu, p.nesterov, p.has_buf);
          if (p.has_buf) *reinterpret_cast<float4*>(bp + (size_t)i * M.n + j) = make_float4(bv[0], bv[1], bv[2], bv[3]);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) ss = fmaf(G[q], G[q], ss);
        put(i, j, G);
      }
      return;
    }
    float gv[8][4], bv[8][4];
    const int j = jb + 4 * lane;
#pragma unroll
    for (int t = 0; t < 8; ++t) {
#pragma unroll
      for (int q = 0; q < 4; ++q) { gv[t][q] = 0.f; bv[t][q] = 0.f; }
      const int i = i0 + 4 * t;
      if (i < M.m && j < M.n) load4((size_t)i * M.n + j, j, M.n, gv[t], bv[t]);
    }
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      const int i = i0 + 4 * t;
      float G[4] = {0.f, 0.f, 0.f, 0.f};
      if (i < M.m && j < M.n) {
#pragma unroll
        for (int q = 0; q < 4; ++q)
          if (j + q < M.n) G[q] = nesterov_g(gv[t][q], bv[t][q], p.mu, p.nesterov, p.has_buf);
        store4((size_t)i * M.n + j, j, M.n, bv[t]);
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) ss = fmaf(G[q], G[q], ss);
      put(i, j, G);
    }
  };
  if (!M.trans) {
    // X = G: rows 0..127 of this CTA's columns c0 .. c0+127
    for (int i0 = warp; i0 < kSmallMaxK; i0 += 32)
      batch(i0, c0, [&](int i, int j, const float (&G)[4]) {
        *reinterpret_cast<uint2*>(Xs + chunk_off((uint32_t)i, (uint32_t)(j - c0))) =
            make_uint2(pack_bf16x2(G[0], G[1]), pack_bf16x2(G[2], G[3]));
      });
  } else {
    // X = G^T: G rows c0 .. c0+127 are this CTA's X columns, G's (<= 128) columns its rows
    for (int i0 = c0 + warp; i0 < c0 + kQuadCols; i0 += 32)
      batch(i0, 0, [&](int i, int j, const float (&G)[4]) {
#pragma unroll
        for (int q = 0; q < 4; ++q)
          *reinterpret_cast<__nv_bfloat16*>(Xs + chunk_off((uint32_t)(j + q), (uint32_t)(i - c0))) =
              __float2bfloat16_rn(G[q]);
      });
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if (lane == 0) red[warp] = ss;
  __syncthreads();
  if (tid < 4) {                                             // this CTA's partial into every CTA's slot
    const float part = red[0] + red[1] + red[2] + red[3];
    st_cluster_u32(mapa_shared(&red[4 + rank], (uint32_t)tid), __float_as_uint(part));
  }
  auto publish = [&]() {                                     // this phase's writes (local and remote) -> next phase
    fence_async_all();
    tc_fence_before();
    cluster_sync_all();
    tc_fence_after();
  };
  auto publish_local = [&]() {                               // this CTA's writes -> its next MMAs
    fence_async_shared();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  };
  publish();
  const float scale =
      1.0f / ((float)sqrt((double)red[4] + (double)red[5] + (double)red[6] + (double)red[7]) + p.eps);
  const uint32_t tmem = *tmem_slot;
  const uint32_t tl = tmem + ((uint32_t)(warp * 32) << 16);  // this warp's 32 lanes
  const int r = warp * 32 + lane;                            // row of X / A / B owned by this thread
  bool ok = true;
  uint32_t phase = 0;
  auto wait_mma = [&]() {
    bool got = ok && mbar_wait(mma_bar, phase, wc, kDevTimeoutAccum);
    phase ^= 1u;
    ok = __syncthreads_and(got) != 0;
    tc_fence_after();
  };
  // W -= lr * O (or O = result) for X columns c0 + 32 cc .. +31 of this thread's
  // row r, staged in the outbox (free by then: the last partials it sent were
  // received before the last rows of A came back; the A buffer may still be
  // the source of this CTA's last bulk copies), then read-modified-written in
  // whole 128-byte rows
  auto apply_chunk = [&](int cc, const float* v) {
    float* S = reinterpret_cast<float*>(outbox);
    if (!M.trans) {
#pragma unroll
      for (int j = 0; j < 8; ++j)
        *reinterpret_cast<float4*>(S + r * 32 + ((j ^ (r & 7)) << 2)) =
            make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
    } else {
#pragma unroll
      for (int q = 0; q < 32; ++q) S[q * 128 + r] = v[q];
    }
    __syncthreads();
    float4 o[8], w4[8];
    float* wp[8];
    bool okw[8], full[8];
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      const int idx = tid + kQuadThreads * t;
      int wi, wj;
      if (!M.trans) {
        const int row = idx >> 3, qd = idx & 7;
        wi = row; wj = c0 + cc * 32 + 4 * qd;
        o[t] = *reinterpret_cast<const float4*>(S + row * 32 + ((qd ^ (row & 7)) << 2));
      } else {
        const int c = idx >> 5, qd = idx & 31;
        wi = c0 + cc * 32 + c; wj = 4 * qd;
        o[t] = *reinterpret_cast<const float4*>(S + c * 128 + 4 * qd);
      }
      okw[t] = wi < M.m && wj < M.n;
      full[t] = M.vec && wj + 3 < M.n;
      wp[t] = M.w + (size_t)wi * M.n + wj;
      w4[t] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (okw[t] && full[t] && !p.assign) w4[t] = *reinterpret_cast<const float4*>(wp[t]);
    }
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      if (!okw[t]) continue;
      if (full[t]) {
        float4 r4 = w4[t];
        if (p.assign) r4 = o[t];
        else { r4.x -= p.lr * o[t].x; r4.y -= p.lr * o[t].y; r4.z -= p.lr * o[t].z; r4.w -= p.lr * o[t].w; }
        *reinterpret_cast<float4*>(wp[t]) = r4;
      } else {
        const float ov[4] = {o[t].x, o[t].y, o[t].z, o[t].w};
        const int wj = (int)((wp[t] - M.w) % M.n);
        for (int e = 0; e < 4 && wj + e < M.n; ++e) wp[t][e] = p.assign ? ov[e] : wp[t][e] - p.lr * ov[e];
      }
    }
    __syncthreads();
  };

  const uint32_t idesc_kk = idesc_bf16_f32(128, 128, 0, 0);
  for (int it = 0; it < p.ns_steps; ++it) {
    const float s = it == 0 ? scale : 1.0f;
    const bool last = it == p.ns_steps - 1;
    // ---- partial Gram of this quarter: P = X_q X_q^T (K = 128 columns)
    if (tid == 0 && ok) {
      // this iteration's incoming bytes: three partials of this CTA's rows and
      // three blocks of rows of A (two 64-column chunks each).  One arrival per
      // phase, and none once the CTA has given up (a phase left incomplete then
      // only collects the bytes of copies already under way, well inside the
      // mbarrier's transaction range)
      mbar_arrive_expect_tx(inbox_bar, 3u * kQuadSlot);
      mbar_arrive_expect_tx(a_bar, 3u * 2u * kQuadARows);
      for (int kk = 0; kk < 8; ++kk) {
        const uint64_t d = smem_desc_sw128(smem_u32(Xs) + (kk >> 2) * kSmallChunk + (kk & 3) * 32, 16, 1024);
        tc_mma_bf16(tmem, d, d, idesc_kk, kk > 0 ? 1u : 0u);
      }
      tc_commit(mma_bar);
    }
    wait_mma();
    if (ok) {
      // row r of P belongs to CTA `warp` (the owner of rows 32 warp .. +31), slot
      // `rank` of its inbox: staged in the slot's layout (in place for this
      // CTA's own rows), then sent by one bulk copy
      const uint32_t w = (uint32_t)warp;
      uint8_t* slot = w == rank ? reinterpret_cast<uint8_t*>(inbox) + rank * kQuadSlot
                                : outbox + (w - (w > rank ? 1u : 0u)) * kQuadSlot;
#pragma unroll 1
      for (int c64 = 0; c64 < 2; ++c64) {
        float v[64];
        tmem_ld_32x32b_x64(tl + (uint32_t)(c64 * 64), v);
#pragma unroll
        for (int q = 0; q < 64; q += 4)
          *reinterpret_cast<float4*>(slot + quad_inbox_off(0u, (uint32_t)lane, (uint32_t)((c64 * 64 + q) >> 2))) =
              make_float4(v[q], v[q + 1], v[q + 2], v[q + 3]);
      }
      // fault injection (debug bit 0): CTA 1 keeps back its first partial for CTA 0,
      // so CTA 0's wait for it runs out, and then every other CTA's wait for CTA 0's rows
      const bool inject_skip = (p.debug_flags & 1) && it == 0 && rank == 1u && w == 0u;
      if (w != rank && !inject_skip) {
        fence_async_shared();                                // the staged rows -> the bulk copy
        __syncwarp();
        if (lane == 0)
          bulk_copy_to_cta(mapa_shared(reinterpret_cast<uint8_t*>(inbox) + rank * kQuadSlot, w), slot, kQuadSlot,
                           mapa_shared(inbox_bar, w));
      }
    }
    {
      // the other CTAs' partials of this CTA's rows have landed (and, through
      // the CTA barrier, this CTA's own slot)
      const bool got = ok && mbar_wait_cluster(inbox_bar, (uint32_t)(it & 1), wc, kDevTimeoutDep);
      ok = __syncthreads_and(got) != 0;
    }
    // ---- rows 32 rank .. +31 of A = s^2 * (P_0 + P_1 + P_2 + P_3), to every CTA
    if (ok) {
      // this thread: row rr of the block, columns 8 j .. 8 j + 7 for j = (tid & 3) + 4 k
      const int rr = tid >> 2;
      const uint8_t* ib = reinterpret_cast<const uint8_t*>(inbox);
      float acc[4][8];
#pragma unroll
      for (int k = 0; k < 4; ++k)
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[k][e] = 0.f;
#pragma unroll
      for (int q = 0; q < 4; ++q)                            // senders in a fixed order
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint32_t j = (uint32_t)((tid & 3) + 4 * k);
          const float4 f0 = *reinterpret_cast<const float4*>(ib + quad_inbox_off((uint32_t)q, (uint32_t)rr, 2 * j));
          const float4 f1 = *reinterpret_cast<const float4*>(ib + quad_inbox_off((uint32_t)q, (uint32_t)rr, 2 * j + 1));
          acc[k][0] += f0.x; acc[k][1] += f0.y; acc[k][2] += f0.z; acc[k][3] += f0.w;
          acc[k][4] += f1.x; acc[k][5] += f1.y; acc[k][6] += f1.z; acc[k][7] += f1.w;
        }
      const int row = (int)rank * 32 + rr;
      const float s2 = s * s;
      uint4 pk[4];
#pragma unroll
      for (int k = 0; k < 4; ++k)
        pk[k] = make_uint4(pack_bf16x2(s2 * acc[k][0], s2 * acc[k][1]), pack_bf16x2(s2 * acc[k][2], s2 * acc[k][3]),
                           pack_bf16x2(s2 * acc[k][4], s2 * acc[k][5]), pack_bf16x2(s2 * acc[k][6], s2 * acc[k][7]));
#pragma unroll
      for (int k = 0; k < 4; ++k)
        *reinterpret_cast<uint4*>(As + chunk_off((uint32_t)row, (uint32_t)(8 * ((tid & 3) + 4 * k)))) = pk[k];
      fence_async_shared();                                  // this CTA's rows of A -> the bulk copies and MMAs
    }
    __syncthreads();
    if (tid == 0 && ok) {
      // rows 32 rank .. +31 of each 64-column chunk: 4 KB at the same place in every CTA
      for (uint32_t d = 1; d < 4; ++d) {
        const uint32_t peer = (rank + d) & 3u;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const uint8_t* src = As + c * kSmallChunk + rank * kQuadARows;
          bulk_copy_to_cta(mapa_shared(src, peer), src, kQuadARows, mapa_shared(a_bar, peer));
        }
      }
    }
    {
      const bool got = ok && mbar_wait_cluster(a_bar, (uint32_t)(it & 1), wc, kDevTimeoutDep);
      ok = __syncthreads_and(got) != 0;
      tc_fence_after();
    }
    // ---- B = b A + c A A (A symmetric: both operands K-major rows of A)
    if (tid == 0 && ok) {
      for (int kk = 0; kk < 8; ++kk) {
        const uint64_t d = smem_desc_sw128(smem_u32(As) + (kk >> 2) * kSmallChunk + (kk & 3) * 32, 16, 1024);
        tc_mma_bf16(tmem, d, d, idesc_kk, kk > 0 ? 1u : 0u);
      }
      tc_commit(mma_bar);
    }
    wait_mma();
#pragma unroll 1
    for (int c64 = 0; c64 < 2 && ok; ++c64) {
      float v[64];
      tmem_ld_32x32b_x64(tl + (uint32_t)(c64 * 64), v);
#pragma unroll
      for (int q = 0; q < 64; q += 8) {
        const uint4 araw = *reinterpret_cast<const uint4*>(As + chunk_off((uint32_t)r, (uint32_t)(c64 * 64 + q)));
        const __nv_bfloat162* ah = reinterpret_cast<const __nv_bfloat162*>(&araw);
        float o8[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(ah[e]);
          o8[2 * e] = fmaf(p.c, v[q + 2 * e], p.b * f.x);
          o8[2 * e + 1] = fmaf(p.c, v[q + 2 * e + 1], p.b * f.y);
        }
        *reinterpret_cast<uint4*>(Bs + chunk_off((uint32_t)r, (uint32_t)(c64 * 64 + q))) =
            make_uint4(pack_bf16x2(o8[0], o8[1]), pack_bf16x2(o8[2], o8[3]), pack_bf16x2(o8[4], o8[5]),
                       pack_bf16x2(o8[6], o8[7]));
      }
    }
    publish_local();
    // ---- X_q' = a s X_q + s B X_q : M = N = K = 128, X read MN-major
    if (tid == 0 && ok) {
      const uint32_t idesc = idesc_bf16_f32(128, 128, 0, 1);
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t a = smem_u32(Bs) + (kk >> 2) * kSmallChunk + (kk & 3) * 32;
        const uint32_t b = smem_u32(Xs) + kk * (16 * 128);
        tc_mma_bf16(tmem, smem_desc_sw128(a, 16, 1024), smem_desc_sw128(b, kSmallChunk, 1024), idesc,
                    kk > 0 ? 1u : 0u);
      }
      tc_commit(mma_bar);
    }
    wait_mma();
#pragma unroll 1
    for (int c64 = 0; c64 < 2 && ok; ++c64) {
      float v64[64];
      tmem_ld_32x32b_x64(tl + (uint32_t)(c64 * 64), v64);
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int cc = 2 * c64 + half;
        float* v = v64 + 32 * half;
#pragma unroll
        for (int q = 0; q < 32; q += 8) {
          const uint32_t xo = chunk_off((uint32_t)r, (uint32_t)(cc * 32 + q));
          const uint4 xraw = *reinterpret_cast<const uint4*>(Xs + xo);
          const __nv_bfloat162* xh = reinterpret_cast<const __nv_bfloat162*>(&xraw);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(xh[e]);
            v[q + 2 * e] = fmaf(s, v[q + 2 * e], p.a * s * f.x);
            v[q + 2 * e + 1] = fmaf(s, v[q + 2 * e + 1], p.a * s * f.y);
          }
          if (!last)
            *reinterpret_cast<uint4*>(Xs + xo) =
                make_uint4(pack_bf16x2(v[q], v[q + 1]), pack_bf16x2(v[q + 2], v[q + 3]),
                           pack_bf16x2(v[q + 4], v[q + 5]), pack_bf16x2(v[q + 6], v[q + 7]));
        }
        if (last) apply_chunk(cc, v);
      }
    }
    if (!last) publish_local();
  }
  if (p.ns_steps == 0 && ok) {
    // O = s * X0 (the listing with an empty loop)
#pragma unroll 1
    for (int cc = 0; cc < kQuadCols / 32; ++cc) {
      float v[32];
#pragma unroll
      for (int q = 0; q < 32; q += 8) {
        const uint4 xraw = *reinterpret_cast<const uint4*>(Xs + chunk_off((uint32_t)r, (uint32_t)(cc * 32 + q)));
        const __nv_bfloat162* xh = reinterpret_cast<const __nv_bfloat162*>(&xraw);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(xh[e]);
          v[q + 2 * e] = scale * f.x;
          v[q + 2 * e + 1] = scale * f.y;
        }
      }
      apply_chunk(cc, v);
    }
  }
  // On the abort path, give bulk copies towards this CTA's shared memory time to
  // land before the cluster leaves (bounded).
  if (!ok || *reinterpret_cast<volatile int*>(abort_flag)) sleep_ns_bounded(200000);
  tc_fence_before();
  cluster_sync_all();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

// ==================================================== bf16 update exchange ===
// For a data-parallel step that exchanges the orthogonalised update O in bf16
// (half the bytes of fp32 weights): `convert` rounds O (fp32, written by a
// step in assign mode) to bf16; `apply` adds -lr * O (bf16) into W.  One CTA
// row per matrix, grid-stride over its elements, 8 elements per thread and
// iteration where both pointers are 16-byte aligned and the count is a
// multiple of 8.
struct O16Args {
  int nmats, apply;
  float lr;
  const float* src[kMaxMats];      // convert: O in fp32
  __nv_bfloat16* o16[kMaxMats];    // convert: destination; apply: O in bf16 (read only)
  float* w[kMaxMats];              // apply: W, updated in place
  long long count[kMaxMats];
  int vec[kMaxMats];
};

__global__ void o16_kernel(const __grid_constant__ O16Args p) {
  griddep_wait();
  const int mi = blockIdx.y;
  if (mi >= p.nmats) return;
  const long long n = p.count[mi];
  const long long stride = (long long)gridDim.x * blockDim.x;
  const long long t0 = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  __nv_bfloat16* o = p.o16[mi];
  if (p.vec[mi]) {
    for (long long e = t0 * 8; e < n; e += stride * 8) {
      if (!p.apply) {
        const float4 a = *reinterpret_cast<const float4*>(p.src[mi] + e);
        const float4 b = *reinterpret_cast<const float4*>(p.src[mi] + e + 4);
        *reinterpret_cast<uint4*>(o + e) = make_uint4(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w),
                                                      pack_bf16x2(b.x, b.y), pack_bf16x2(b.z, b.w));
      } else {
        const uint4 raw = *reinterpret_cast<const uint4*>(o + e);
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
        float4* wp = reinterpret_cast<float4*>(p.w[mi] + e);
        float4 a = wp[0], b = wp[1];
        const float2 h0 = __bfloat1622float2(h[0]), h1 = __bfloat1622float2(h[1]);
        const float2 h2 = __bfloat1622float2(h[2]), h3 = __bfloat1622float2(h[3]);
        a.x = fmaf(-p.lr, h0.x, a.x); a.y = fmaf(-p.lr, h0.y, a.y);
        a.z = fmaf(-p.lr, h1.x, a.z); a.w = fmaf(-p.lr, h1.y, a.w);
        b.x = fmaf(-p.lr, h2.x, b.x); b.y = fmaf(-p.lr, h2.y, b.y);
        b.z = fmaf(-p.lr, h3.x, b.z); b.w = fmaf(-p.lr, h3.y, b.w);
        wp[0] = a;
        wp[1] = b;
      }
    }
  } else {
    for (long long e = t0; e < n; e += stride) {
      if (!p.apply) o[e] = __float2bfloat16_rn(p.src[mi][e]);
      else p.w[mi][e] = fmaf(-p.lr, __bfloat162float(o[e]), p.w[mi][e]);
    }
  }
}

// ======================================================= ns_steps == 0 ===
__global__ void apply_x0_kernel(const __grid_constant__ ApplyArgs p) {
  griddep_wait();
  const int mi = blockIdx.y;
  if (mi >= p.nmats) return;
  const OutMat& O = p.out[mi];
  const float s = p.scale[mi];
  const size_t total = (size_t)O.m * O.n;
  for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (size_t)gridDim.x * blockDim.x) {
    const int i = (int)(e / O.n), j = (int)(e % O.n);
    const size_t xi = O.trans ? ((size_t)j * p.lp[mi] + i) : ((size_t)i * p.lp[mi] + j);
    const float v = s * __bfloat162float(p.x[mi][xi]);
    O.w[e] = p.assign ? v : O.w[e] - p.lr * v;
  }
}

}  // namespace muon
