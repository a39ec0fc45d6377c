// Device kernels of the Muon step (Modded-NanoGPT article, "Muon optimizer"
// section: Nesterov momentum, then zeroth_power_via_newtonschulz5, then the
// weight update).
//
//   prologue_kernel   buf <- mu*buf + g ; G = g + mu*buf ; per-matrix ||G||_F ;
//                     X0 = bf16(G), stored short-side-major (k x l, padded).
//   ns_gemm_kernel    one persistent tcgen05 GEMM launch per NS phase over all
//                     matrices of a group:
//                       GRAM    A = s^2 * X X^T            (upper tiles, mirrored)
//                       POLY    B = b*A + c*(A A)          (upper tiles, mirrored)
//                       UPDATE  X' = a*s*X + s*(B X)       (last step: W -= lr*X')
//                     s = 1/(||G||_F+eps) on the first iteration, 1 afterwards,
//                     so the listing's normalisation is folded into epilogues.
//   apply_x0_kernel   ns_steps == 0: W -= lr * s * X0.
#pragma once

#include <cuda.h>
#include "ptx.cuh"

namespace muon {

constexpr int kBM = 128;            // tile rows (TMEM lanes)
constexpr int kBN = 128;            // tile cols (TMEM fp32 columns per accumulator)
constexpr int kBK = 64;             // K per pipeline stage: one 128-byte swizzle row of bf16
constexpr int kUmmaK = 16;          // K of one tcgen05.mma kind::f16
constexpr int kStages = 4;
constexpr int kGemmThreads = 192;   // warp 0 TMA, warp 1 MMA (+TMEM alloc), warps 2..5 epilogue
constexpr int kEpiThreads = 128;
constexpr int kTmemCols = 256;      // two 128-column fp32 accumulators
constexpr int kMaxClasses = 16;
constexpr int kMaxMats = 320;
constexpr int kTmapsPerClass = 6;
constexpr int kPad = 128;           // padding granule of the short and long sides

enum TmapSlot : int { kTmX0 = 0, kTmX1 = 1, kTmX0mn = 2, kTmX1mn = 3, kTmA = 4, kTmB = 5 };
enum GemmMode : int { kModeGram = 0, kModePoly = 1, kModeUpdate = 2 };

constexpr uint32_t kStageABytes = kBM * kBK * 2;     // 16 KB
constexpr uint32_t kStageBBytes = kBN * kBK * 2;     // 16 KB
constexpr uint32_t kStageBytes = kStageABytes + kStageBBytes;
constexpr uint32_t kTileBytes = kBM * kBN * 2;       // 32 KB bf16 output / epilogue input tile
constexpr uint32_t kChunkBytes = kBM * 64 * 2;       // 16 KB: 128 rows x 64 cols (one TMA box)
constexpr uint32_t kSmemDataBytes = kStages * kStageBytes + 2 * kTileBytes;
constexpr uint32_t kSmemCtrlBytes = 256;
constexpr uint32_t kGemmSmemBytes = kSmemDataBytes + kSmemCtrlBytes + 1024;  // + alignment slack

// ------------------------------------------------------------ arguments ---
struct GemmClass {
  int batch;          // matrices of this shape class
  int kp, lp;         // padded short side (rows of X) and long side (cols of X)
  int mat_first;      // first matrix of the class in group order
  int tiles_m;        // kp / 128
  int tiles_n;        // UPDATE: lp / 128; GRAM / POLY: tiles_m
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

struct GemmArgs {
  const CUtensorMap* tmaps;
  const CUtensorMap* wmaps;   // per matrix (group order): W as fp32 [m][n]; box 32x128 (X = W) or 32x32 (X = W^T)
  const float* scale;     // per matrix (group order): 1/(||G||_F + eps)
  int* status;
  unsigned long long wait_limit_ns;
  int nclasses, total_tiles;
  int mode, x_in, first, final_apply, assign, debug_flags;
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

  const int t = blockIdx.x;
  const int mi = find_mat(p, t);
  const ProMat& M = p.mats[mi];
  const int local = t - M.tile_begin;
  const int xr0 = (local / M.tiles_c) * kProRows;
  const int xc0 = (local % M.tiles_c) * kProCols;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  float ss = 0.f;

  if (!M.trans) {
    // X[xr][xc] = G[xr][xc]: each warp walks one row segment of 128 columns.
#pragma unroll 2
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
#pragma unroll 2
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

// Byte offset of the 16-byte unit u (0..7) of row r inside a 128-row x 128-byte
// box stored with the 128-byte swizzle (the pattern TMA writes / reads).
__device__ __forceinline__ uint32_t sw128_off(uint32_t r, uint32_t u) { return r * 128u + ((u ^ (r & 7u)) << 4); }

// Read-modify-write of one 128 x 32 slice of the final result into W (or
// O), staged in shared memory by the epilogue.  X row gi0 + r, col gj0 + c maps
// to W[gi][gj] (X = W) or W[gj][gi] (X = W^T).  Each warp touches whole rows.
__device__ __forceinline__ void store_w_slice(const OutMat& O, const float* S, int gi0, int gj0, int et, float lr,
                                              int assign) {
  // all loads of the slice are issued before any store (8 in flight per thread)
  float4 o[8], w[8];
  float* wp[8];
  bool ok[8], full[8];
#pragma unroll
  for (int it = 0; it < 8; ++it) {
    int row, col, sidx;
    if (!O.trans) {
      const int rr = it * 16 + (et >> 3), q = et & 7;
      row = gi0 + rr; col = gj0 + 4 * q;
      sidx = rr * 32 + ((q ^ (rr & 7)) << 2);
      ok[it] = row < O.m && col < O.n;
    } else {
      const int c = it * 4 + (et >> 5), q = et & 31;
      row = gj0 + c; col = gi0 + 4 * q;          // W[row][col..col+3]
      sidx = c * kBM + 4 * q;
      ok[it] = row < O.m && col < O.n;
    }
    full[it] = O.vec && col + 3 < O.n;
    wp[it] = O.w + (size_t)row * O.n + col;
    o[it] = *reinterpret_cast<const float4*>(S + sidx);
    w[it] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (ok[it] && full[it] && !assign) w[it] = *reinterpret_cast<const float4*>(wp[it]);
  }
  const float sg = assign ? -1.f : lr;
#pragma unroll
  for (int it = 0; it < 8; ++it) {
    if (!ok[it]) continue;
    if (full[it]) {
      float4 r4 = w[it];
      r4.x -= sg * o[it].x; r4.y -= sg * o[it].y; r4.z -= sg * o[it].z; r4.w -= sg * o[it].w;
      *reinterpret_cast<float4*>(wp[it]) = r4;
    } else {
      const float ov[4] = {o[it].x, o[it].y, o[it].z, o[it].w};
      const int col = (int)((wp[it] - O.w) % O.n);
      for (int e = 0; e < 4 && col + e < O.n; ++e) wp[it][e] = assign ? ov[e] : wp[it][e] - lr * ov[e];
    }
  }
}

struct __align__(8) GemmCtrl {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t tmem_full[2];
  uint64_t tmem_empty[2];
  uint64_t dfull;
  uint64_t dempty;
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

__global__ void __launch_bounds__(kGemmThreads, 1) ns_gemm_kernel(const __grid_constant__ GemmArgs p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stage_base = smem;
  uint8_t* dtile = smem + kStages * kStageBytes;       // epilogue input tile / output staging
  uint8_t* mtile = dtile + kTileBytes;                 // mirrored (transposed) output staging
  GemmCtrl* ctl = reinterpret_cast<GemmCtrl*>(mtile + kTileBytes);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool sym = p.mode != kModeUpdate;
  const bool has_d = p.mode != kModeGram;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) { mbar_init(&ctl->full[s], 1); mbar_init(&ctl->empty[s], 1); }
    for (int s = 0; s < 2; ++s) { mbar_init(&ctl->tmem_full[s], 1); mbar_init(&ctl->tmem_empty[s], kEpiThreads); }
    mbar_init(&ctl->dfull, 1);
    mbar_init(&ctl->dempty, 1);
    mbar_init(&ctl->drain, 1);
    ctl->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&ctl->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = ctl->tmem_base;
  WaitCtx wc{&ctl->abort_flag, p.status, p.wait_limit_ns};

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    if (lane == 0) {
      for (int c = 0; c < p.nclasses; ++c)
        for (int k = 0; k < kTmapsPerClass; ++k) {
          const CUtensorMap* tm = &p.tmaps[p.cls[c].tmap_base + k];
          tmap_acquire(tm);
          tmap_prefetch(tm);
        }
      int stage = 0;
      uint32_t phase = 0;
      int pending[kStages];            // parity of the last issued, not yet landed, fill (-1: none)
      for (int s = 0; s < kStages; ++s) pending[s] = -1;
      int dpending = -1;
      bool ok = true;
      int it = 0;
      for (int t = blockIdx.x; t < p.total_tiles && ok; t += gridDim.x, ++it) {
        const TileCoord tc = decode_tile(p, t, sym);
        const GemmClass& C = p.cls[tc.cls];
        const CUtensorMap* tA;
        const CUtensorMap* tB;
        if (p.mode == kModeGram) { tA = &p.tmaps[C.tmap_base + (p.x_in ? kTmX1 : kTmX0)]; tB = tA; }
        else if (p.mode == kModePoly) { tA = &p.tmaps[C.tmap_base + kTmA]; tB = tA; }
        else { tA = &p.tmaps[C.tmap_base + kTmB]; tB = &p.tmaps[C.tmap_base + (p.x_in ? kTmX1mn : kTmX0mn)]; }
        for (int kb = 0; kb < C.kblocks; ++kb) {
          if (!mbar_wait(&ctl->empty[stage], phase ^ 1u, wc, kDevTimeoutEmpty)) { ok = false; break; }
          uint8_t* sa = stage_base + stage * kStageBytes;
          uint8_t* sb = sa + kStageABytes;
          const bool inject_skip = (p.debug_flags & 1) && it == 0 && kb == 0;
          if (!inject_skip) {
            mbar_arrive_expect_tx(&ctl->full[stage], kStageBytes);
            tma_load_3d(sa, tA, &ctl->full[stage], kb * kBK, tc.tm * kBM, tc.b);
            if (p.mode == kModeUpdate) {
              // B operand = X rows [kb*64, +64) x cols [tn*128, +128), MN-major: two 64-col boxes
              tma_load_3d(sb, tB, &ctl->full[stage], tc.tn * kBN, kb * kBK, tc.b);
              tma_load_3d(sb + kStageBBytes / 2, tB, &ctl->full[stage], tc.tn * kBN + 64, kb * kBK, tc.b);
            } else {
              tma_load_3d(sb, tB, &ctl->full[stage], kb * kBK, tc.tn * kBN, tc.b);
            }
            pending[stage] = (int)phase;
          }
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        if (has_d) {
          if (!mbar_wait(&ctl->dempty, (uint32_t)((it & 1) ^ 1), wc, kDevTimeoutEpi)) { ok = false; break; }
          const CUtensorMap* tD = (p.mode == kModePoly) ? &p.tmaps[C.tmap_base + kTmA]
                                                        : &p.tmaps[C.tmap_base + (p.x_in ? kTmX1 : kTmX0)];
          mbar_arrive_expect_tx(&ctl->dfull, kTileBytes);
          tma_load_3d(dtile, tD, &ctl->dfull, tc.tn * kBN, tc.tm * kBM, tc.b);
          tma_load_3d(dtile + kChunkBytes, tD, &ctl->dfull, tc.tn * kBN + 64, tc.tm * kBM, tc.b);
          dpending = it & 1;
        }
      }
      // Never leave the CTA with copies in flight into its shared memory.
      for (int s = 0; s < kStages; ++s)
        if (pending[s] >= 0) mbar_wait(&ctl->full[s], (uint32_t)pending[s], wc, kDevTimeoutDrain);
      if (dpending >= 0) mbar_wait(&ctl->dfull, (uint32_t)dpending, wc, kDevTimeoutDrain);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(kBM, kBN, 0, p.mode == kModeUpdate ? 1 : 0);
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      bool issued_any = false;
      for (int t = blockIdx.x; t < p.total_tiles && ok; t += gridDim.x, ++it) {
        const TileCoord tc = decode_tile(p, t, sym);
        const GemmClass& C = p.cls[tc.cls];
        const int acc = it & 1;
        const uint32_t acc_phase = (uint32_t)((it >> 1) & 1);
        if (!mbar_wait(&ctl->tmem_empty[acc], acc_phase ^ 1u, wc, kDevTimeoutAccum)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * kBN);
        for (int kb = 0; kb < C.kblocks; ++kb) {
          if (!mbar_wait(&ctl->full[stage], phase, wc, kDevTimeoutFull)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_u32(stage_base + stage * kStageBytes);
          const uint32_t sb = sa + kStageABytes;
#pragma unroll
          for (int kk = 0; kk < kBK / kUmmaK; ++kk) {
            const uint64_t adesc = smem_desc_sw128(sa + kk * (kUmmaK * 2), 16, 1024);
            const uint64_t bdesc = (p.mode == kModeUpdate)
                                       ? smem_desc_sw128(sb + kk * (kUmmaK * 128), kStageBBytes / 2, 1024)
                                       : smem_desc_sw128(sb + kk * (kUmmaK * 2), 16, 1024);
            tc_mma_bf16(d_tmem, adesc, bdesc, idesc, (kb | kk) != 0 ? 1u : 0u);
          }
          issued_any = true;
          tc_commit(&ctl->empty[stage]);
          if (++stage == kStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        tc_commit(&ctl->tmem_full[acc]);
      }
      if (issued_any) {                 // all MMAs done before TMEM is released
        tc_commit(&ctl->drain);
        mbar_wait(&ctl->drain, 0, wc, kDevTimeoutDrain);
      }
    }
  } else {
    // --------------------------------------------------------- epilogue
    const int et = threadIdx.x - 64;              // 0..127
    const int q = warp & 3;                       // TMEM lane quarter this warp may access
    const int r = q * 32 + lane;                  // tile row owned by this thread
    const float alpha_first = 1.0f;
    if (et == 0) {
      for (int c = 0; c < p.nclasses; ++c)
        for (int k = 0; k < kTmapsPerClass; ++k) tmap_acquire(&p.tmaps[p.cls[c].tmap_base + k]);
      if (p.mode == kModeUpdate && p.final_apply)
        for (int c = 0; c < p.nclasses; ++c)
          for (int b = 0; b < p.cls[c].batch; ++b)
            if (p.out[p.cls[c].mat_first + b].tma) tmap_acquire(&p.wmaps[p.cls[c].mat_first + b]);
    }
    int it = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < p.total_tiles; t += gridDim.x, ++it) {
      const TileCoord tc = decode_tile(p, t, sym);
      const GemmClass& C = p.cls[tc.cls];
      const int mat = C.mat_first + tc.b;
      const int acc = it & 1;
      const uint32_t acc_phase = (uint32_t)((it >> 1) & 1);
      if (ok) ok = mbar_wait(&ctl->tmem_full[acc], acc_phase, wc, kDevTimeoutAccum);
      tc_fence_after();
      if (ok && has_d) ok = mbar_wait(&ctl->dfull, (uint32_t)(it & 1), wc, kDevTimeoutEpi);
      // one outcome for all 128 epilogue threads: the branch below holds named
      // barriers and warp-collective tcgen05.ld
      ok = named_bar_and(1, kEpiThreads, ok);
      const float s = p.first ? p.scale[mat] : alpha_first;
      const bool mirror = sym && tc.tm != tc.tn;
      const bool final_w = p.mode == kModeUpdate && p.final_apply;
      if (ok) {
        const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * kBN);
#pragma unroll 1
        for (int cc = 0; cc < kBN / 32; ++cc) {
          float v[32];
          tmem_ld_32x32b_x32(tbase + (uint32_t)(cc * 32), v);
          const int h = cc >> 1;                          // 64-column chunk
          uint8_t* drow = dtile + h * kChunkBytes;
          if (p.mode == kModeGram) {
            const float alpha = s * s;
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] *= alpha;
          } else {
            // epilogue input (A for POLY, X for UPDATE): 4 units of 8 bf16
            const float wd = (p.mode == kModePoly) ? p.b : p.a * s;
            const float wa = (p.mode == kModePoly) ? p.c : s;
#pragma unroll
            for (int uu = 0; uu < 4; ++uu) {
              const uint32_t u = (uint32_t)((cc & 1) * 4 + uu);
              uint4 raw = *reinterpret_cast<const uint4*>(drow + sw128_off((uint32_t)r, u));
              const __nv_bfloat162* hv = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                float2 f = __bfloat1622float2(hv[e]);
                v[uu * 8 + 2 * e] = fmaf(wa, v[uu * 8 + 2 * e], wd * f.x);
                v[uu * 8 + 2 * e + 1] = fmaf(wa, v[uu * 8 + 2 * e + 1], wd * f.y);
              }
            }
          }
          if (final_w && p.out[mat].tma) {
            // -lr*O (or O) for a 128 x 32 slice, staged 128-byte swizzled; TMA adds
            // it to W in L2 (or stores it), so W never passes through the SM.
            const OutMat& O = p.out[mat];
            const float sg = p.assign ? 1.f : -p.lr;
            uint8_t* S = mtile + (cc & 1) * kChunkBytes;
            if (!O.trans) {
#pragma unroll
              for (int j = 0; j < 8; ++j)
                *reinterpret_cast<float4*>(S + sw128_off((uint32_t)r, (uint32_t)j)) =
                    make_float4(sg * v[4 * j], sg * v[4 * j + 1], sg * v[4 * j + 2], sg * v[4 * j + 3]);
            } else {
              // box h = r / 32 holds W rows gj0..gj0+31 x W cols gi0+32h..+31
              uint8_t* Sh = S + (r >> 5) * 4096;
              const int rr = r & 31;
#pragma unroll
              for (int i = 0; i < 32; ++i)
                *reinterpret_cast<float*>(Sh + sw128_off((uint32_t)i, (uint32_t)(rr >> 2)) + (rr & 3) * 4) =
                    sg * v[i];
            }
            fence_async_shared();
            named_bar_sync(1, kEpiThreads);
            if (et == 0) {
              const CUtensorMap* wm = &p.wmaps[mat];
              const int gi0 = tc.tm * kBM, gj0 = tc.tn * kBN + cc * 32;
              if (!O.trans) {
                if (p.assign) tma_store_2d(wm, S, gj0, gi0); else tma_reduce_add_2d(wm, S, gj0, gi0);
              } else {
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                  if (p.assign) tma_store_2d(wm, S + h * 4096, gi0 + 32 * h, gj0);
                  else tma_reduce_add_2d(wm, S + h * 4096, gi0 + 32 * h, gj0);
                }
              }
              tma_store_commit();
              tma_store_wait_read1();          // the other staging buffer is free again
            }
            named_bar_sync(1, kEpiThreads);
          } else if (final_w) {
            // fp32 result slice (128 rows x 32 cols) through shared memory so that
            // W is read and written in whole 128-byte rows.
            const OutMat& O = p.out[mat];
            float* S = reinterpret_cast<float*>(mtile + (cc & 1) * (kChunkBytes));
            if (!O.trans) {
              // S[row][quad ^ (row & 7)]: 8 float4 per row
#pragma unroll
              for (int j = 0; j < 8; ++j)
                *reinterpret_cast<float4*>(S + r * 32 + ((j ^ (r & 7)) << 2)) =
                    make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
            } else {
              // S[col][row]: row c of S is a 128-float row of W
#pragma unroll
              for (int i = 0; i < 32; ++i) S[i * kBM + r] = v[i];
            }
            named_bar_sync(1, kEpiThreads);
            store_w_slice(O, S, tc.tm * kBM, tc.tn * kBN + cc * 32, et, p.lr, p.assign);
          } else {
            // bf16 output tile (in place over the input tile), 128-byte swizzled for the TMA store
#pragma unroll
            for (int uu = 0; uu < 4; ++uu) {
              const uint32_t u = (uint32_t)((cc & 1) * 4 + uu);
              uint4 o;
              o.x = pack_bf16x2(v[uu * 8 + 0], v[uu * 8 + 1]);
              o.y = pack_bf16x2(v[uu * 8 + 2], v[uu * 8 + 3]);
              o.z = pack_bf16x2(v[uu * 8 + 4], v[uu * 8 + 5]);
              o.w = pack_bf16x2(v[uu * 8 + 6], v[uu * 8 + 7]);
              *reinterpret_cast<uint4*>(drow + sw128_off((uint32_t)r, u)) = o;
            }
            if (mirror) {
              // transposed copy: row c of the mirror tile holds column c of this tile
              uint8_t* mchunk = mtile + (r >> 6) * kChunkBytes;
              const uint32_t mu = (uint32_t)((r & 63) >> 3);
#pragma unroll
              for (int i = 0; i < 32; ++i) {
                const uint32_t crow = (uint32_t)(cc * 32 + i);
                __nv_bfloat16* dst =
                    reinterpret_cast<__nv_bfloat16*>(mchunk + sw128_off(crow, mu)) + (r & 7);
                *dst = __float2bfloat16_rn(v[i]);
              }
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&ctl->tmem_empty[acc]);
      fence_async_shared();
      named_bar_sync(1, kEpiThreads);
      if (et == 0 && ok && !final_w) {
        const CUtensorMap* tO;
        if (p.mode == kModeGram) tO = &p.tmaps[C.tmap_base + kTmA];
        else if (p.mode == kModePoly) tO = &p.tmaps[C.tmap_base + kTmB];
        else tO = &p.tmaps[C.tmap_base + (p.x_in ? kTmX0 : kTmX1)];
        tma_store_3d(tO, dtile, tc.tn * kBN, tc.tm * kBM, tc.b);
        tma_store_3d(tO, dtile + kChunkBytes, tc.tn * kBN + 64, tc.tm * kBM, tc.b);
        if (mirror) {
          tma_store_3d(tO, mtile, tc.tm * kBM, tc.tn * kBN, tc.b);
          tma_store_3d(tO, mtile + kChunkBytes, tc.tm * kBM + 64, tc.tn * kBN, tc.b);
        }
        tma_store_commit();
        tma_store_wait_read0();
      }
      named_bar_sync(1, kEpiThreads);
      if (et == 0 && has_d) mbar_arrive(&ctl->dempty);
    }
    if (et == 0) tma_store_wait_all0();
  }

  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// ======================================================= ns_steps == 0 ===
__global__ void apply_x0_kernel(const __grid_constant__ ApplyArgs p) {
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
