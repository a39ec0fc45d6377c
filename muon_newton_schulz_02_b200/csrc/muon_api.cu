// Host side of the C ABI declared in include/muon.h.
//
// A call is planned once per set of shapes: matrices are grouped into shape
// classes (same padded short side kp and long side lp), each class gets
// contiguous [batch][kp][lp] bf16 iterates and [batch][kp][kp] Gram /
// polynomial buffers in the workspace, and one TMA descriptor per buffer and
// box shape.  A step of a group is then the fused momentum/norm/cast prologue
// and either one chained persistent tcgen05 GEMM launch that runs every
// Newton-Schulz phase and the weight update from host-built work lists (short
// sides up to 1024), or one launch per phase (3 * ns_steps launches), all on
// the caller's stream.  Small matrices (short side <= 128, long side <= 512;
// or both sides <= 256, run by CTA pairs) need no workspace: one launch of a
// fused kernel runs their whole step.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <cmath>
#include <atomic>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <list>
#include <map>
#include <memory>
#include <mutex>
#include <queue>
#include <set>
#include <string>
#include <vector>

#include "muon.h"
#include "kernels.cuh"

using namespace muon;

namespace {

thread_local std::string g_last_error = "no error";
std::mutex g_mu;
std::atomic<int64_t> g_launches{0};
bool g_profile = false;
int g_debug_flags = 0;
uint64_t g_wait_limit_ns = 2000000000ull;

int fail(int code, const std::string& msg) {
  g_last_error = msg;
  return code;
}

#define CUDA_TRY(expr)                                                                        \
  do {                                                                                        \
    cudaError_t e_ = (expr);                                                                  \
    if (e_ != cudaSuccess) return fail(MUON_ERR_CUDA, std::string(#expr) + ": " + cudaGetErrorString(e_)); \
  } while (0)

size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }
int round_up(int v, int a) { return (v + a - 1) / a * a; }

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// ------------------------------------------------------------------ plan ---
struct MatDesc {
  int m, n, k, l, kp, lp, trans;
  int user;                 // index in the caller's arrays
};

struct ClassDesc {
  int kp, lp;
  std::vector<int> mats;    // group-order indices
  size_t off_x0, off_x1, off_a, off_b;
  size_t off_x8 = 0, off_a8 = 0;   // e4m3 copies of X and A (muon_step_fp8 only), past every other region
};

struct Group {
  std::vector<MatDesc> mats;     // group order (class by class)
  std::vector<ClassDesc> classes;
  std::vector<int> pro_tile_begin;
  int pro_tiles = 0;
  size_t off_partials = 0, off_tickets = 0, off_scale = 0, off_done = 0, off_tmaps = 0, off_wmaps = 0;
  size_t off_tmaps8 = 0;           // in Plan::tmaps8
  size_t data_bytes = 0;
  int sym_tiles = 0, upd_tiles = 0;
  std::vector<GemmClass> sym_cls, upd_cls;
  std::vector<size_t> guards;      // guard-band offsets (MUON_GUARD_BANDS=1), kGuardBytes each
};

// The first kTicketBytes of every workspace hold the per-matrix arrival
// counters of the prologue's norm reduction.  They are zeroed when the
// workspace is allocated and every prologue leaves them at zero again, so no
// plan may place anything else there.
constexpr size_t kTicketBytes = 4096;
static_assert(kMaxMats * 4 <= kTicketBytes, "ticket region too small");

// Guard bands (a debugging aid, MUON_GUARD_BANDS=1 in the environment when the
// library is loaded): kGuardBytes of a fixed byte after every workspace region
// of a group, written before the group's launches; muon_guard_check reports
// any byte a launch changed, i.e. a write past the end of a region.
constexpr size_t kGuardBytes = 4096;
constexpr unsigned char kGuardByte = 0xA5;
bool guard_bands() {
  static int on = -1;
  if (on < 0) {
    const char* e = std::getenv("MUON_GUARD_BANDS");
    on = (e && std::atoi(e) != 0) ? 1 : 0;
  }
  return on == 1;
}

// Work lists of one chained launch (see ns_gemm_kernel<..., true>) for one
// group and one iteration count, in device memory: the items of every
// cluster back to back, then the cluster offsets.
struct ChainTables {
  int nclusters = 0;
  int nitems = 0;
  void* dev = nullptr;
  const WorkItem* items = nullptr;
  const int* off = nullptr;
};

constexpr int kWmapRing = 4;

struct Plan {
  std::vector<int64_t> shapes;
  std::vector<Group> groups;
  std::vector<MatDesc> small;               // matrices of the fused single-CTA kernel (no workspace)
  std::vector<MatDesc> pair;                // matrices of the fused CTA-pair kernel (no workspace)
  std::vector<MatDesc> quad;                // matrices of the fused four-CTA kernel (no workspace)
  size_t ws_bytes = 0;
  size_t ws_bytes_fp8 = 0;                  // with the e4m3 copies of muon_step_fp8
  size_t tmap_bytes = 0;
  size_t tmap8_bytes = 0;
  void* ws = nullptr;                       // workspace the tensor maps point into
  void* tmaps = nullptr;                    // this plan's own device copy of its tensor maps
  void* tmaps8 = nullptr;                   // tensor maps of the e4m3 copies, encoded by the first fp8 call
  // Per group: fp32 tensor maps of the caller's output matrices, re-encoded
  // when the caller passes other pointers; host copies in a ring of
  // kWmapRing pinned staging slots, so that re-encoding does not wait for the
  // upload of the previous call (the chunks of muon_step_host reuse plans).
  std::vector<std::vector<const void*>> wmap_key;
  std::vector<CUtensorMap*> wmap_host;      // per group: kWmapRing slots of its matrices' maps
  cudaEvent_t wmap_copied[kWmapRing] = {};  // per slot: its last upload has been read
  int wmap_next = 0;
  std::map<std::pair<size_t, int>, ChainTables> chains;   // (group, ns_steps) -> work lists
  ~Plan() {
    if (tmaps) cudaFree(tmaps);
    if (tmaps8) cudaFree(tmaps8);
    for (auto& kv : chains)
      if (kv.second.dev) cudaFree(kv.second.dev);
    for (auto h : wmap_host)
      if (h) cudaFreeHost(h);
    for (auto e : wmap_copied)
      if (e) cudaEventDestroy(e);
  }
};

// Splits the matrices into groups (each within the per-launch limits) and lays
// out each group's workspace; groups run one after another and share the
// data region, each keeps its own tensor-map table at the end.
int build_layout(const int64_t* shapes, int n, Plan& plan) {
  plan.shapes.assign(shapes, shapes + 2 * (size_t)n);
  std::vector<MatDesc> all(n);
  for (int i = 0; i < n; ++i) {
    const int64_t m = shapes[2 * i], c = shapes[2 * i + 1];
    if (m <= 0 || c <= 0) return fail(MUON_ERR_SHAPE, "matrix " + std::to_string(i) + " has a dimension <= 0");
    if (m > (1 << 20) || c > (1 << 20) || m * c > (int64_t(1) << 31))
      return fail(MUON_ERR_SHAPE, "matrix " + std::to_string(i) + " is too large (dims <= 2^20, elements <= 2^31)");
    MatDesc d;
    d.m = (int)m; d.n = (int)c;
    d.trans = m > c ? 1 : 0;
    d.k = (int)std::min(m, c); d.l = (int)std::max(m, c);
    d.kp = round_up(d.k, kPad); d.lp = round_up(d.l, kPad);
    if (d.kp > 16384) return fail(MUON_ERR_SHAPE, "short side above 16384 is not supported");
    d.user = i;
    all[i] = d;
  }
  // short side <= 128 and long side <= 512: fused single-CTA kernel, no workspace
  {
    std::vector<MatDesc> big;
    for (const auto& d : all) {
      if (d.k <= kSmallMaxK && round_up(d.l, 64) <= kSmallMaxL) plan.small.push_back(d);
      else if (d.k <= kPairMaxK && d.l <= kPairMaxL) plan.pair.push_back(d);
      else big.push_back(d);
    }
    all.swap(big);
    // A few such matrices with a long side above 256 leave most SMs idle under
    // one CTA each: they take a cluster of four CTAs (a quarter of the long
    // side each) instead.  Many of them fill the GPU one CTA each already.
    int longer = 0;
    for (const auto& d : plan.small) longer += d.l > 256;
    if (longer > 0 && longer <= kQuadMaxMats) {
      std::vector<MatDesc> keep;
      for (const auto& d : plan.small) (d.l > 256 ? plan.quad : keep).push_back(d);
      plan.small.swap(keep);
    }
  }
  // greedy grouping in caller order, respecting kMaxMats and kMaxClasses
  std::vector<std::vector<MatDesc>> raw;
  {
    std::vector<MatDesc> cur;
    std::vector<std::pair<int, int>> keys;
    for (const auto& d : all) {
      const std::pair<int, int> key(d.kp, d.lp);
      const bool new_key = std::find(keys.begin(), keys.end(), key) == keys.end();
      if ((int)cur.size() == kMaxMats || (new_key && (int)keys.size() == kMaxClasses)) {
        raw.push_back(cur); cur.clear(); keys.clear();
      }
      if (std::find(keys.begin(), keys.end(), key) == keys.end()) keys.push_back(key);
      cur.push_back(d);
    }
    if (!cur.empty()) raw.push_back(cur);
  }
  size_t data_max = 0;
  for (auto& gm : raw) {
    Group g;
    g.off_tickets = 0;          // fixed region, see kTicketBytes
    // classes ordered by decreasing long side (longest GEMM K first)
    std::map<std::pair<int, int>, std::vector<MatDesc>> by;
    for (const auto& d : gm) by[{-d.lp, -d.kp}].push_back(d);
    size_t off = kTicketBytes;
    // the next region starts at `off`; `end` is the end of the one just placed
    auto place = [&](size_t end) {
      off = align_up(end, 1024);
      if (guard_bands()) { g.guards.push_back(off); off += kGuardBytes; }
    };
    place(off);
    for (auto& kv : by) {
      ClassDesc c;
      c.kp = -kv.first.second; c.lp = -kv.first.first;
      const size_t batch = kv.second.size();
      const size_t xb = batch * (size_t)c.kp * c.lp * 2, ab = batch * (size_t)c.kp * c.kp * 2;
      c.off_x0 = off; place(off + xb);
      c.off_x1 = off; place(off + xb);
      c.off_a = off; place(off + ab);
      c.off_b = off; place(off + ab);
      for (auto& d : kv.second) { c.mats.push_back((int)g.mats.size()); g.mats.push_back(d); }
      g.classes.push_back(c);
    }
    for (const auto& d : g.mats) {
      g.pro_tile_begin.push_back(g.pro_tiles);
      g.pro_tiles += (d.kp / kProRows) * (d.lp / kProCols);
    }
    g.off_partials = off; place(off + (size_t)g.pro_tiles * 4);
    g.off_scale = off; place(off + g.mats.size() * 4);
    g.off_done = off; place(off + g.mats.size() * 4);
    g.data_bytes = off;
    data_max = std::max(data_max, off);
    // GEMM tile bookkeeping
    int sym = 0, upd = 0, first = 0;
    for (size_t ci = 0; ci < g.classes.size(); ++ci) {
      const ClassDesc& c = g.classes[ci];
      GemmClass s{}, u{};
      s.batch = u.batch = (int)c.mats.size();
      s.kp = u.kp = c.kp; s.lp = u.lp = c.lp;
      s.mat_first = u.mat_first = first;
      s.tiles_m = u.tiles_m = (c.kp + kTile - 1) / kTile;
      s.tiles_n = s.tiles_m;
      u.tiles_n = (c.lp + kTile - 1) / kTile;
      s.tiles_per_mat = s.tiles_m * (s.tiles_m + 1) / 2;
      u.tiles_per_mat = u.tiles_m * u.tiles_n;
      s.tile_begin = sym; u.tile_begin = upd;
      sym += s.tiles_per_mat * s.batch;
      upd += u.tiles_per_mat * u.batch;
      s.kblocks = c.lp / kBK;   // GRAM; POLY overrides with kp / 64
      u.kblocks = c.kp / kBK;
      s.tmap_base = u.tmap_base = (int)ci * kTmapsPerClass;
      first += (int)c.mats.size();
      g.sym_cls.push_back(s);
      g.upd_cls.push_back(u);
    }
    g.sym_tiles = sym; g.upd_tiles = upd;
    plan.groups.push_back(std::move(g));
  }
  size_t off = 0;
  for (auto& g : plan.groups) {
    g.off_tmaps = off;
    off = align_up(off + g.classes.size() * kTmapsPerClass * sizeof(CUtensorMap), 1024);
    g.off_wmaps = off;
    off = align_up(off + g.mats.size() * sizeof(CUtensorMap), 1024);
  }
  plan.tmap_bytes = off;
  plan.ws_bytes = data_max;
  // e4m3 copies of X and A (muon_step_fp8) after everything else, so that
  // the bf16 path's layout and size do not depend on them
  plan.ws_bytes_fp8 = data_max;
  off = 0;
  for (auto& g : plan.groups) {
    size_t o = align_up(data_max, 1024);
    for (auto& cd : g.classes) {
      const size_t batch = cd.mats.size();
      cd.off_x8 = o; o = align_up(o + batch * (size_t)cd.kp * cd.lp, 1024);
      cd.off_a8 = o; o = align_up(o + batch * (size_t)cd.kp * cd.kp, 1024);
    }
    plan.ws_bytes_fp8 = std::max(plan.ws_bytes_fp8, o);
    g.off_tmaps8 = off;
    off = align_up(off + g.classes.size() * kTmaps8PerClass * sizeof(CUtensorMap), 1024);
  }
  plan.tmap8_bytes = off;
  return MUON_OK;
}

// ------------------------------------------------------ chained schedule ---
// Host-side list scheduling of the chained launch.  Every matrix runs the
// chain Gram(0), poly(0), update(0), Gram(1), ..., update(n-1) (the last
// update adds -lr*O into W); each phase's tiles may start only once all tiles
// of the previous phase of that matrix are done.  A simulation of `ncl` clusters
// assigns tiles greedily: a free cluster takes the next tile of the
// highest-priority matrix whose current phase is ready (longest remaining
// critical path first), so a matrix's phases follow each other closely, its
// operands stay in L2 while other matrices fill the gaps, and the matrices
// finish together instead of leaving a tail of dependent phases with too few
// tiles to keep every cluster busy.  Tile cost is modelled as its K-blocks
// plus a fixed overhead; a finished tile is visible to dependants `lat` units
// later (epilogue, store, and the producer running ahead of the MMAs).
//
// Each cluster's list is in order of simulated start time, and every item's
// inputs come from items with strictly earlier simulated start times, so with
// all clusters resident some list head can always proceed: the lists cannot
// deadlock.  `need` counts tile halves (each CTA of a pair publishes its own).
double chain_latency_units() {
  static double lat = -1.0;
  if (lat < 0.0) {
    const char* e = std::getenv("MUON_CHAIN_LATENCY");
    lat = e ? std::max(0.0, std::atof(e)) : 20.0;
  }
  return lat;
}

bool chain_static_priority() {
  static int rule = -1;
  if (rule < 0) {
    const char* e = std::getenv("MUON_CHAIN_PRIORITY");
    rule = (e && std::strcmp(e, "static") == 0) ? 1 : 0;
  }
  return rule == 1;
}

void build_chain(const Group& g, int ns_steps, int ncl, std::vector<WorkItem>& items, std::vector<int>& off) {
  constexpr double kOverhead = 2.0;
  constexpr double kFinalCost = 1.5;          // the last update also reads and writes W
  const double lat = chain_latency_units();
  const int nm = (int)g.mats.size();
  const int nphases = 3 * ns_steps;
  struct MatState {
    int cls = 0, b = 0, T = 0, Tn = 0;
    int ntiles[4] = {0, 0, 0, 0};
    double cost[4] = {0, 0, 0, 0};
    int phase = 0, next = 0;
    int need = 0;              // tile halves completed before the current phase
    double vis = 0.0;          // latest visibility time among the current phase's tiles
    double total = 0.0;
  };
  auto mode_of = [&](int j) { return j == nphases - 1 ? (int)kModeFinal : j % 3; };
  auto cost_of = [&](const auto& st, int j) { return st.cost[mode_of(j)]; };
  std::vector<MatState> ms(nm);
  for (size_t ci = 0; ci < g.classes.size(); ++ci) {
    const ClassDesc& cd = g.classes[ci];
    for (size_t b = 0; b < cd.mats.size(); ++b) {
      MatState& st = ms[cd.mats[b]];
      st.cls = (int)ci;
      st.b = (int)b;
      st.T = (cd.kp + kTile - 1) / kTile;
      st.Tn = (cd.lp + kTile - 1) / kTile;
      st.ntiles[kModeGram] = st.ntiles[kModePoly] = st.T * (st.T + 1) / 2;
      st.ntiles[kModeUpdate] = st.ntiles[kModeFinal] = st.T * st.Tn;
      st.cost[kModeGram] = cd.lp / kBK + kOverhead;
      st.cost[kModePoly] = st.cost[kModeUpdate] = cd.kp / kBK + kOverhead;
      st.cost[kModeFinal] = kFinalCost * st.cost[kModeUpdate];
      for (int j = 0; j < nphases; ++j) st.total += st.ntiles[mode_of(j)] * cost_of(st, j);
    }
  }
  // Priority of a matrix whose next phase is ready: by default the longest
  // remaining critical path (one tile plus the visibility latency per phase
  // still to run) first, so that the matrices finish together and no long
  // chain is left alone at the end; "static": more total work first.
  std::vector<int> by_prio(nm);
  for (int i = 0; i < nm; ++i) by_prio[i] = i;
  std::stable_sort(by_prio.begin(), by_prio.end(), [&](int x, int y) { return ms[x].total > ms[y].total; });
  std::vector<int> prio(nm);
  for (int r = 0; r < nm; ++r) prio[by_prio[r]] = r;
  const bool static_rule = chain_static_priority();
  std::vector<double> key(nm, 0.0);           // the key a matrix holds while its phase is available
  auto key_of = [&](int m) {
    if (static_rule) return (double)prio[m];
    double path = 0.0;
    for (int q = ms[m].phase; q < nphases; ++q) path += cost_of(ms[m], q) + lat;
    return -path;
  };

  std::vector<std::vector<WorkItem>> lists(ncl);
  std::priority_queue<std::pair<double, int>, std::vector<std::pair<double, int>>, std::greater<>> free_at;
  for (int c = 0; c < ncl; ++c) free_at.push({0.0, c});
  std::set<std::pair<double, int>> pending;   // (ready time, matrix) of a matrix's next phase
  std::set<std::pair<double, int>> avail;     // (key, matrix): matrices with ready, unassigned tiles, best first
  auto make_avail = [&](int m) {
    key[m] = key_of(m);
    avail.insert({key[m], m});
  };
  for (int m = 0; m < nm; ++m)
    if (nphases > 0) make_avail(m);
  long long left = 0;
  for (int m = 0; m < nm; ++m)
    for (int j = 0; j < nphases; ++j) left += ms[m].ntiles[mode_of(j)];
  while (left > 0) {
    auto [t, c] = free_at.top();
    free_at.pop();
    auto admit = [&](double now) {
      while (!pending.empty() && pending.begin()->first <= now) {
        make_avail(pending.begin()->second);
        pending.erase(pending.begin());
      }
    };
    admit(t);
    if (avail.empty()) {                      // this cluster idles until a phase becomes ready
      t = std::max(t, pending.begin()->first);
      admit(t);
    }
    const int m = avail.begin()->second;
    MatState& st = ms[m];
    const int mode = mode_of(st.phase);
    int tm, tn;
    if (mode == kModeUpdate || mode == kModeFinal) {
      tm = st.next / st.Tn;
      tn = st.next % st.Tn;
    } else {                                  // upper-triangle 256-blocks, row by row
      int r = st.next, row = 0, len = st.T;
      while (r >= len) { r -= len; ++row; --len; }
      tm = row;
      tn = row + r;
    }
    WorkItem w{};
    w.need = st.need;
    w.mat = (unsigned short)m;
    w.b = (unsigned short)st.b;
    w.tm = (unsigned short)tm;
    w.tn = (unsigned short)tn;
    w.cls = (unsigned char)st.cls;
    w.mode = (unsigned char)mode;
    w.it = (unsigned short)(st.phase / 3);
    lists[c].push_back(w);
    const double end = t + cost_of(st, st.phase);
    st.vis = std::max(st.vis, end + lat);
    free_at.push({end, c});
    --left;
    if (++st.next == st.ntiles[mode]) {       // phase fully assigned: the next one is ready at st.vis
      avail.erase({key[m], m});
      st.need += 2 * st.ntiles[mode];
      st.next = 0;
      if (++st.phase < nphases) pending.insert({st.vis, m});
      st.vis = 0.0;
    }
  }
  items.clear();
  off.assign(1, 0);
  for (int c = 0; c < ncl; ++c) {
    items.insert(items.end(), lists[c].begin(), lists[c].end());
    off.push_back((int)items.size());
  }
}

// [batch][rows][cols] tensor of bf16 (esize 2) or e4m3 bytes (esize 1).
int encode_map(CUtensorMap* map, void* base, int cols, int rows, int batch, int box_cols, int box_rows,
               int esize = 2, CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B) {
  auto fn = encode_fn();
  if (!fn) return fail(MUON_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  cuuint64_t dims[3] = {(cuuint64_t)cols, (cuuint64_t)rows, (cuuint64_t)batch};
  cuuint64_t strides[2] = {(cuuint64_t)cols * esize, (cuuint64_t)cols * rows * esize};
  cuuint32_t box[3] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows, 1};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = fn(map, esize == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, base, dims,
                  strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MUON_ERR_CUDA, "cuTensorMapEncodeTiled failed: " + std::to_string((int)r));
  return MUON_OK;
}

// The tensor maps of one shape class's e4m3 copies (see Tmap8Slot).
int encode_class_maps8(CUtensorMap* m, char* base, const ClassDesc& cd) {
  const int batch = (int)cd.mats.size();
  int rc;
  if ((rc = encode_map(&m[kTm8X], base + cd.off_x8, cd.lp, cd.kp, batch, 128, 128, 1))) return rc;
  if ((rc = encode_map(&m[kTm8A], base + cd.off_a8, cd.kp, cd.kp, batch, 128, 128, 1))) return rc;
  if ((rc = encode_map(&m[kTm8Xs], base + cd.off_x8, cd.lp, cd.kp, batch, 64, 128, 1, CU_TENSOR_MAP_SWIZZLE_64B)))
    return rc;
  if ((rc = encode_map(&m[kTm8As], base + cd.off_a8, cd.kp, cd.kp, batch, 64, 128, 1, CU_TENSOR_MAP_SWIZZLE_64B)))
    return rc;
  return MUON_OK;
}

// The 8 tensor maps of one shape class (see TmapSlot) over its buffers at `base`.
int encode_class_maps(CUtensorMap* m, char* base, const ClassDesc& cd) {
  const int batch = (int)cd.mats.size();
  int rc;
  if ((rc = encode_map(&m[kTmX0], base + cd.off_x0, cd.lp, cd.kp, batch, 64, 128))) return rc;
  if ((rc = encode_map(&m[kTmX1], base + cd.off_x1, cd.lp, cd.kp, batch, 64, 128))) return rc;
  if ((rc = encode_map(&m[kTmX0mn], base + cd.off_x0, cd.lp, cd.kp, batch, 64, 64))) return rc;
  if ((rc = encode_map(&m[kTmX1mn], base + cd.off_x1, cd.lp, cd.kp, batch, 64, 64))) return rc;
  if ((rc = encode_map(&m[kTmA], base + cd.off_a, cd.kp, cd.kp, batch, 64, 128))) return rc;
  if ((rc = encode_map(&m[kTmB], base + cd.off_b, cd.kp, cd.kp, batch, 64, 128))) return rc;
  if ((rc = encode_map(&m[kTmAmn], base + cd.off_a, cd.kp, cd.kp, batch, 64, 64))) return rc;
  if ((rc = encode_map(&m[kTmBmn], base + cd.off_b, cd.kp, cd.kp, batch, 64, 64))) return rc;
  return MUON_OK;
}

// Launch with programmatic stream serialization: the kernel may be scheduled
// while the previous launch on the stream drains; it calls griddepcontrol.wait
// before touching anything the previous launch wrote.
template <class Args>
cudaError_t launch_pdl(void (*kernel)(Args), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       const Args& args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args);
}

// One GEMM launch: persistent clusters of two CTAs (one CTA per SM).  With
// `chain_clusters` > 0 it is the chained launch over that many clusters (every
// phase and the weight update); otherwise one Newton-Schulz phase (args.mode).
cudaError_t launch_gemm(cudaStream_t stream, const GemmArgs& args, int sm_count, int chain_clusters = 0) {
  const int pairs = chain_clusters > 0 ? chain_clusters : std::max(1, std::min(args.total_tiles, sm_count / 2));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs, 1, 1);
  cfg.blockDim = dim3(kGemmThreads, 1, 1);
  cfg.dynamicSmemBytes = chain_clusters > 0 ? kChainSmemBytes : kGemmSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  // e4m3 instantiations only for the per-phase launches that use them (the last update never does)
  const bool f8 = args.fp8_iters > 0 && args.iter < args.fp8_iters;
  if (chain_clusters > 0) return cudaLaunchKernelEx(&cfg, ns_gemm_kernel<kModeGram, false, true>, args);
  switch (args.mode) {
    case kModeGram:
      return f8 ? cudaLaunchKernelEx(&cfg, ns_gemm_kernel<kModeGram, false, false, true>, args)
                : cudaLaunchKernelEx(&cfg, ns_gemm_kernel<kModeGram, false, false>, args);
    case kModePoly:
      return f8 ? cudaLaunchKernelEx(&cfg, ns_gemm_kernel<kModePoly, false, false, true>, args)
                : cudaLaunchKernelEx(&cfg, ns_gemm_kernel<kModePoly, false, false>, args);
    default:
      if (args.final_apply) return cudaLaunchKernelEx(&cfg, ns_gemm_kernel<kModeUpdate, true, false>, args);
      return f8 ? cudaLaunchKernelEx(&cfg, ns_gemm_kernel<kModeUpdate, false, false, true>, args)
                : cudaLaunchKernelEx(&cfg, ns_gemm_kernel<kModeUpdate, false, false>, args);
  }
}

// W (m x n fp32, row-major, n % 4 == 0, 16-byte aligned) as a 2-D tensor map
// for the final epilogue: box 32 cols x 128 rows (X = W) or 32 x 32 (X = W^T).
int encode_wmap(CUtensorMap* map, void* w, int m, int n, int trans) {
  auto fn = encode_fn();
  if (!fn) return fail(MUON_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  cuuint64_t dims[2] = {(cuuint64_t)n, (cuuint64_t)m};
  cuuint64_t strides[1] = {(cuuint64_t)n * 4};
  cuuint32_t box[2] = {32, trans ? 32u : 128u};
  cuuint32_t es[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, w, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(MUON_ERR_CUDA, "cuTensorMapEncodeTiled (W) failed: " + std::to_string((int)r));
  return MUON_OK;
}

// ---------------------------------------------------------------- context ---
struct ProfRec { int kind; cudaEvent_t a, b; };

struct Ctx {
  int dev = 0;
  cudaStream_t stream = nullptr;
  void* ws = nullptr;
  size_t ws_cap = 0;
  std::list<std::unique_ptr<Plan>> plans;   // most recent first
  int* status_h = nullptr;
  int* status_d = nullptr;
  float* stage = nullptr;                   // device staging of muon_step_host
  float* o32 = nullptr;                     // fp32 O of muon_update_bf16 before its rounding to bf16
  size_t o32_cap = 0;
  size_t stage_cap = 0;
  std::vector<ProfRec> prof;
  std::vector<cudaEvent_t> event_pool;
  int sm_count = 148;
  cudaStream_t h2d = nullptr, d2h = nullptr;       // copy streams of muon_step_host
  std::vector<cudaEvent_t> host_events;            // per-chunk ordering events of muon_step_host
  std::vector<size_t> guards;                      // guard bands of the last group run (MUON_GUARD_BANDS=1)
};

std::map<std::pair<int, void*>, std::unique_ptr<Ctx>> g_ctx;
std::map<int, bool> g_dev_ready;
std::map<int, int> g_chain_clusters;      // per device: clusters of two CTAs that can be resident at once

int device_setup(int dev) {
  if (g_dev_ready[dev]) return MUON_OK;
  cudaDeviceProp prop;
  CUDA_TRY(cudaGetDeviceProperties(&prop, dev));
  if (prop.major != 10 || prop.minor != 0)
    return fail(MUON_ERR_DEVICE, "this library is built for sm_100a (B200); device is sm_" +
                                     std::to_string(prop.major) + std::to_string(prop.minor));
  CUDA_TRY(cudaFuncSetAttribute(ns_small_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmallSmem));
  CUDA_TRY(cudaFuncSetAttribute(ns_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kPairSmem));
  CUDA_TRY(cudaFuncSetAttribute(ns_quad_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kQuadSmem));
  CUDA_TRY(cudaFuncSetAttribute(ns_gemm_kernel<kModeGram, false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)kGemmSmemBytes));
  CUDA_TRY(cudaFuncSetAttribute(ns_gemm_kernel<kModePoly, false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)kGemmSmemBytes));
  CUDA_TRY(cudaFuncSetAttribute(ns_gemm_kernel<kModeUpdate, false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)kGemmSmemBytes));
  CUDA_TRY(cudaFuncSetAttribute(ns_gemm_kernel<kModeUpdate, true, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)kGemmSmemBytes));
  CUDA_TRY(cudaFuncSetAttribute(ns_gemm_kernel<kModeGram, false, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)kChainSmemBytes));
  CUDA_TRY(cudaFuncSetAttribute(ns_gemm_kernel<kModeGram, false, false, true>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kGemmSmemBytes));
  CUDA_TRY(cudaFuncSetAttribute(ns_gemm_kernel<kModePoly, false, false, true>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kGemmSmemBytes));
  CUDA_TRY(cudaFuncSetAttribute(ns_gemm_kernel<kModeUpdate, false, false, true>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kGemmSmemBytes));

  {
    // The chained launch's clusters wait on one another's results, so all of
    // them must be resident at once: never launch more than the device holds.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(prop.multiProcessorCount, 1, 1);
    cfg.blockDim = dim3(kGemmThreads, 1, 1);
    cfg.dynamicSmemBytes = kChainSmemBytes;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int nclusters = 0;
    if (cudaOccupancyMaxActiveClusters(&nclusters, (void*)ns_gemm_kernel<kModeGram, false, true>, &cfg) !=
        cudaSuccess) {
      cudaGetLastError();
      nclusters = 0;                         // chained launch unavailable: one launch per phase
    }
    g_chain_clusters[dev] = std::min(nclusters, prop.multiProcessorCount / 2);
  }
  g_dev_ready[dev] = true;
  return MUON_OK;
}

int get_ctx(void* stream, Ctx** out) {
  int dev = 0;
  CUDA_TRY(cudaGetDevice(&dev));
  int rc = device_setup(dev);
  if (rc) return rc;
  auto key = std::make_pair(dev, stream);
  auto it = g_ctx.find(key);
  if (it == g_ctx.end()) {
    auto c = std::make_unique<Ctx>();
    c->dev = dev;
    c->stream = (cudaStream_t)stream;
    CUDA_TRY(cudaHostAlloc((void**)&c->status_h, sizeof(int), cudaHostAllocMapped));
    *c->status_h = 0;
    CUDA_TRY(cudaHostGetDevicePointer((void**)&c->status_d, c->status_h, 0));
    CUDA_TRY(cudaDeviceGetAttribute(&c->sm_count, cudaDevAttrMultiProcessorCount, dev));
    it = g_ctx.emplace(key, std::move(c)).first;
  }
  *out = it->second.get();
  return MUON_OK;
}

int ensure_workspace(Ctx& c, size_t bytes) {
  if (c.ws_cap >= bytes) return MUON_OK;
  CUDA_TRY(cudaStreamSynchronize(c.stream));
  if (c.ws) { cudaFree(c.ws); c.ws = nullptr; c.ws_cap = 0; }
  c.plans.clear();                                     // their tensor maps point into the old workspace
  const size_t cap = align_up(bytes, size_t(1) << 21);
  if (cudaMalloc(&c.ws, cap) != cudaSuccess) {
    cudaGetLastError();
    return fail(MUON_ERR_NOMEM, "workspace allocation of " + std::to_string(cap) + " bytes failed");
  }
  c.ws_cap = cap;
  CUDA_TRY(cudaMemset(c.ws, 0, cap));                  // tickets start at zero
  return MUON_OK;
}

constexpr size_t kMaxPlans = 48;

// Tensor maps of the plan's e4m3 copies (muon_step_fp8), encoded on first use.
int ensure_fp8_maps(Plan& p) {
  if (p.tmaps8 || !p.tmap8_bytes) return MUON_OK;
  void* d = nullptr;
  if (cudaMalloc(&d, p.tmap8_bytes) != cudaSuccess) {
    cudaGetLastError();
    return fail(MUON_ERR_NOMEM, "tensor-map table allocation failed");
  }
  for (auto& g : p.groups) {
    std::vector<CUtensorMap> maps(g.classes.size() * kTmaps8PerClass);
    int rc = MUON_OK;
    for (size_t ci = 0; ci < g.classes.size() && !rc; ++ci)
      rc = encode_class_maps8(&maps[ci * kTmaps8PerClass], (char*)p.ws, g.classes[ci]);
    if (!rc && cudaMemcpy((char*)d + g.off_tmaps8, maps.data(), maps.size() * sizeof(CUtensorMap),
                          cudaMemcpyHostToDevice) != cudaSuccess) {
      const cudaError_t e = cudaGetLastError();
      rc = fail(MUON_ERR_CUDA, std::string("tensor-map upload failed: ") + cudaGetErrorString(e));
    }
    if (rc) {
      cudaFree(d);
      return rc;
    }
  }
  p.tmaps8 = d;
  return MUON_OK;
}

// The plan of these shapes, built on first use; `fp8`: the workspace must also
// hold the e4m3 copies and their tensor maps must exist.
int get_plan(Ctx& c, const int64_t* shapes, int n, Plan** out, bool fp8 = false) {
  for (auto it = c.plans.begin(); it != c.plans.end(); ++it) {
    Plan& p = **it;
    if ((int)p.shapes.size() == 2 * n && std::memcmp(p.shapes.data(), shapes, sizeof(int64_t) * 2 * n) == 0 &&
        p.ws == c.ws && (!fp8 || c.ws_cap >= p.ws_bytes_fp8)) {
      c.plans.splice(c.plans.begin(), c.plans, it);
      *out = c.plans.front().get();
      return fp8 ? ensure_fp8_maps(**out) : MUON_OK;
    }
  }
  auto p = std::make_unique<Plan>();
  int rc = build_layout(shapes, n, *p);
  if (rc) return rc;
  rc = ensure_workspace(c, std::max<size_t>(fp8 ? p->ws_bytes_fp8 : p->ws_bytes, kTicketBytes));
  if (rc) return rc;
  p->ws = c.ws;
  char* base = (char*)c.ws;
  if (p->tmap_bytes && cudaMalloc(&p->tmaps, p->tmap_bytes) != cudaSuccess) {
    cudaGetLastError();
    p->tmaps = nullptr;
    return fail(MUON_ERR_NOMEM, "tensor-map table allocation failed");
  }
  for (auto& g : p->groups) {
    std::vector<CUtensorMap> maps(g.classes.size() * kTmapsPerClass);
    for (size_t ci = 0; ci < g.classes.size(); ++ci) {
      if ((rc = encode_class_maps(&maps[ci * kTmapsPerClass], base, g.classes[ci]))) return rc;
    }
    CUDA_TRY(cudaMemcpy((char*)p->tmaps + g.off_tmaps, maps.data(), maps.size() * sizeof(CUtensorMap),
                        cudaMemcpyHostToDevice));
  }
  p->wmap_key.resize(p->groups.size());
  p->wmap_host.assign(p->groups.size(), nullptr);
  for (size_t gi = 0; gi < p->groups.size(); ++gi) {
    if (cudaHostAlloc((void**)&p->wmap_host[gi], kWmapRing * p->groups[gi].mats.size() * sizeof(CUtensorMap),
                      cudaHostAllocDefault) != cudaSuccess) {
      cudaGetLastError();
      p->wmap_host[gi] = nullptr;
      return fail(MUON_ERR_NOMEM, "pinned tensor-map staging allocation failed");
    }
  }
  for (auto& e : p->wmap_copied) CUDA_TRY(cudaEventCreateWithFlags(&e, cudaEventDisableTiming));
  c.plans.push_front(std::move(p));
  // Keep the most recent kMaxPlans plans: enough for the chunks of the
  // host-buffer entry point (up to 16 shape lists) next to the device-buffer
  // calls of the same loop, so that no steady-state call rebuilds a plan.
  if (c.plans.size() > kMaxPlans) {
    CUDA_TRY(cudaStreamSynchronize(c.stream));
    while (c.plans.size() > kMaxPlans) c.plans.pop_back();
  }
  *out = c.plans.front().get();
  return fp8 ? ensure_fp8_maps(**out) : MUON_OK;
}

// ---------------------------------------------------------------- launches ---
cudaEvent_t pool_event(Ctx& c) {
  if (!c.event_pool.empty()) {
    cudaEvent_t e = c.event_pool.back();
    c.event_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

// NVTX range names of the launch kinds (MUON_KIND_*), for timeline tools; the
// ranges cost nothing when no tool is attached.
const char* const kKindNames[MUON_NUM_KINDS] = {"muon.prologue", "muon.gram", "muon.poly", "muon.update",
                                                "muon.update_apply", "muon.apply_x0", "muon.small", "muon.pair",
                                                "muon.chain", "muon.o16", "muon.quad"};

template <class F>
int launch(Ctx& c, int kind, F&& f) {
  cudaEvent_t e0 = nullptr, e1 = nullptr;
  if (g_profile) {
    e0 = pool_event(c);
    e1 = pool_event(c);
    cudaEventRecord(e0, c.stream);
  }
  nvtxRangePushA(kKindNames[kind]);
  f();
  nvtxRangePop();
  cudaError_t err = cudaGetLastError();
  if (g_profile) {
    cudaEventRecord(e1, c.stream);
    c.prof.push_back({kind, e0, e1});
  }
  if (err != cudaSuccess) return fail(MUON_ERR_CUDA, std::string("kernel launch failed: ") + cudaGetErrorString(err));
  g_launches.fetch_add(1);
  return MUON_OK;
}

struct StepIO {
  float* const* W;          // outputs (W, or O when assign)
  const float* const* g;
  float* const* buf;        // may be null (no momentum)
  float lr, mu, a, b, c, eps;
  int ns_steps, nesterov, assign;
  int fp8_iters = 0;        // muon_step_fp8: iterations with e4m3 operands (0: bf16 throughout)
};

// Power-of-two scale that maps magnitudes up to `bound` into e4m3's finite
// range (|x| <= 448), with a margin for the bf16 rounding of what is bounded.
float e4m3_scale(double bound) {
  const double e = std::floor(std::log2(448.0 / (1.0625 * std::max(bound, 1e-30))));
  return std::ldexp(1.0f, (int)std::min(60.0, std::max(-60.0, e)));
}

// Scales of the e4m3 copies of X_i and A_i for quintic coefficients (a, b, c).
// The normalised first iterate has singular values in [0, 1]; an iterate whose
// singular values lie in [0, r] has a Gram matrix with eigenvalues in [0, r^2]
// and a successor with singular values |sigma q(sigma^2)|, q(x) = a + b x +
// c x^2.  Every entry of a matrix is at most its largest singular value, so
// these bounds (maximised on a fine grid, with the margin above) keep the
// copies finite.
void e4m3_scales(float a, float b, float c, float* sx8, float* sa8) {
  auto q = [&](double x) { return a + b * x + c * x * x; };
  auto pmax = [&](double r) {                // max |sigma q(sigma^2)| over [0, r]
    double m = 0.0;
    for (int i = 0; i <= 4096; ++i) {
      const double sg = r * i / 4096.0;
      m = std::max(m, std::fabs(sg * q(sg * sg)));
    }
    return m;
  };
  double r = 1.0;
  for (int i = 0; i < kMaxFp8Iters; ++i) {
    sx8[i] = e4m3_scale(r);
    sa8[i] = e4m3_scale(r * r);
    r = pmax(r);
  }
}

// The error a device status code reports (`what`: the launches it came from).
int status_error(int s, const std::string& what) {
  if (s == kDevBounds)
    return fail(MUON_ERR_DEVICE, what + " met a tile outside its class, matrix or tile grid (device bounds check, "
                                        "code " + std::to_string(s) + ")");
  return fail(MUON_ERR_TIMEOUT, what + " gave up on a bounded wait (device code " + std::to_string(s) + ")");
}

int check_status(Ctx& c) {
  const int s = *(volatile int*)c.status_h;
  if (s != 0) {
    *(volatile int*)c.status_h = 0;
    return status_error(s, "an earlier launch on this stream");
  }
  return MUON_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Encodes and uploads the output tensor maps of group gi if the caller's
// output pointers differ from the ones encoded last time.
int update_wmaps(Ctx& c, Plan& plan, size_t gi, const StepIO& io) {
  const Group& g = plan.groups[gi];
  std::vector<const void*> key(g.mats.size());
  for (size_t i = 0; i < g.mats.size(); ++i) key[i] = io.W[g.mats[i].user];
  if (key == plan.wmap_key[gi]) return MUON_OK;
  const int slot = plan.wmap_next;
  plan.wmap_next = (slot + 1) % kWmapRing;
  CUDA_TRY(cudaEventSynchronize(plan.wmap_copied[slot]));   // this slot's previous upload was read
  CUtensorMap* h = plan.wmap_host[gi] + (size_t)slot * g.mats.size();
  std::memset(h, 0, g.mats.size() * sizeof(CUtensorMap));
  for (size_t i = 0; i < g.mats.size(); ++i) {
    const MatDesc& d = g.mats[i];
    void* w = (void*)io.W[d.user];
    if (d.n % 4 == 0 && aligned16(w)) {
      int rc = encode_wmap(&h[i], w, d.m, d.n, d.trans);
      if (rc) return rc;
    }
  }
  CUDA_TRY(cudaMemcpyAsync((char*)plan.tmaps + g.off_wmaps, h, g.mats.size() * sizeof(CUtensorMap),
                           cudaMemcpyHostToDevice, c.stream));
  CUDA_TRY(cudaEventRecord(plan.wmap_copied[slot], c.stream));
  plan.wmap_key[gi] = key;
  return MUON_OK;
}

constexpr int kChainMaxK = 1024;       // largest padded short side the chained launch takes
constexpr int64_t kChainMaxItems = int64_t(1) << 22;   // largest work list (64 MiB of items)

// Work items of the chained launch for group g: every tile of every phase.
int64_t chain_items(const Group& g, int ns_steps) {
  int64_t per_iter = 0;
  for (const auto& cd : g.classes) {
    const int64_t T = (cd.kp + kTile - 1) / kTile, Tn = (cd.lp + kTile - 1) / kTile;
    per_iter += (int64_t)cd.mats.size() * (T * (T + 1) + T * Tn);   // Gram + polynomial + update
  }
  return per_iter * ns_steps;
}

// The chained launch's work lists for group gidx and ns_steps iterations,
// built and uploaded on first use (a synchronous copy: make the first call for
// a set of shapes and an iteration count outside stream capture).
int get_chain(Ctx& c, Plan& plan, size_t gidx, int ns_steps, ChainTables** out) {
  const auto key = std::make_pair(gidx, ns_steps);
  auto it = plan.chains.find(key);
  if (it == plan.chains.end()) {
    ChainTables ct;
    ct.nclusters = g_chain_clusters[c.dev];
    std::vector<WorkItem> items;
    std::vector<int> off;
    build_chain(plan.groups[gidx], ns_steps, ct.nclusters, items, off);
    ct.nitems = (int)items.size();
    const size_t ib = align_up(items.size() * sizeof(WorkItem), 256), ob = off.size() * sizeof(int);
    if (cudaMalloc(&ct.dev, ib + ob) != cudaSuccess) {
      cudaGetLastError();
      return fail(MUON_ERR_NOMEM, "work-list allocation failed");
    }
    if (cudaMemcpy(ct.dev, items.data(), items.size() * sizeof(WorkItem), cudaMemcpyHostToDevice) != cudaSuccess ||
        cudaMemcpy((char*)ct.dev + ib, off.data(), ob, cudaMemcpyHostToDevice) != cudaSuccess) {
      const cudaError_t e = cudaGetLastError();
      cudaFree(ct.dev);
      return fail(MUON_ERR_CUDA, std::string("work-list upload failed: ") + cudaGetErrorString(e));
    }
    ct.items = (const WorkItem*)ct.dev;
    ct.off = (const int*)((char*)ct.dev + ib);
    it = plan.chains.emplace(key, ct).first;   // owned by the plan from here on
  }
  *out = &it->second;
  return MUON_OK;
}

int run_group(Ctx& c, Plan& plan, size_t gidx, const StepIO& io) {
  const Group& g = plan.groups[gidx];
  char* base = (char*)c.ws;
  float* scale = (float*)(base + g.off_scale);
  const CUtensorMap* tmaps = (const CUtensorMap*)((char*)plan.tmaps + g.off_tmaps);
  const int nm = (int)g.mats.size();
  unsigned* done = (unsigned*)(base + g.off_done);
  // every phase in one chained launch, unless the device cannot hold its
  // clusters, a test asks for one launch per phase, or the matrices are so
  // large that one phase of one matrix already fills the GPU (short side above
  // kChainMaxK): there the phases gain little from overlapping, and keeping
  // several such matrices in flight costs more L2 misses than it saves.
  bool chain = io.ns_steps >= 1 && g_chain_clusters[c.dev] > 0 && !(g_debug_flags & 4);
  for (const auto& cd : g.classes) chain = chain && cd.kp <= kChainMaxK;
  chain = chain && chain_items(g, io.ns_steps) <= kChainMaxItems;   // lists of bounded size and build time

  if (guard_bands()) {
    for (size_t off : g.guards) CUDA_TRY(cudaMemsetAsync(base + off, kGuardByte, kGuardBytes, c.stream));
    c.guards = g.guards;
  }

  // 1. prologue
  {
    auto pa = std::make_unique<ProArgs>();
    std::memset(pa.get(), 0, sizeof(ProArgs));
    pa->nmats = nm;
    pa->total_tiles = g.pro_tiles;
    pa->mu = io.mu;
    pa->eps = io.eps;
    pa->nesterov = io.nesterov;
    pa->has_buf = io.buf != nullptr;
    pa->partials = (float*)(base + g.off_partials);
    pa->tickets = (unsigned*)(base + g.off_tickets);
    pa->scale = scale;
    pa->done = chain ? done : nullptr;
    for (const auto& cd : g.classes) {
      for (size_t b = 0; b < cd.mats.size(); ++b) {
        const int gi = cd.mats[b];
        const MatDesc& d = g.mats[gi];
        ProMat& pm = pa->mats[gi];
        pm.g = io.g[d.user];
        pm.buf = io.buf ? io.buf[d.user] : nullptr;
        pm.x = (__nv_bfloat16*)(base + cd.off_x0 + b * (size_t)cd.kp * cd.lp * 2);
        pm.m = d.m; pm.n = d.n; pm.kp = d.kp; pm.lp = d.lp;
        pm.trans = d.trans;
        pm.vec = (d.n % 4 == 0) && aligned16(pm.g) && (!pm.buf || aligned16(pm.buf));
        pm.tile_begin = g.pro_tile_begin[gi];
        pm.tiles_c = d.lp / kProCols;
        pm.tiles = (d.kp / kProRows) * pm.tiles_c;
      }
    }
    int rc = launch(c, MUON_KIND_PROLOGUE,
                    [&] { launch_pdl(prologue_kernel, dim3(g.pro_tiles), dim3(kProThreads), 0, c.stream, *pa); });
    if (rc) return rc;
  }

  auto fill_out = [&](OutMat* out) {
    for (const auto& cd : g.classes)
      for (size_t b = 0; b < cd.mats.size(); ++b) {
        const int gi = cd.mats[b];
        const MatDesc& d = g.mats[gi];
        OutMat& o = out[gi];
        o.w = io.W[d.user];
        o.m = d.m; o.n = d.n; o.trans = d.trans;
        o.vec = (d.n % 4 == 0) && aligned16(o.w);
        o.tma = o.vec;
      }
  };

  if (io.ns_steps == 0) {
    auto aa = std::make_unique<ApplyArgs>();
    std::memset(aa.get(), 0, sizeof(ApplyArgs));
    aa->scale = scale;
    aa->lr = io.lr;
    aa->assign = io.assign;
    aa->nmats = nm;
    fill_out(aa->out);
    for (const auto& cd : g.classes)
      for (size_t b = 0; b < cd.mats.size(); ++b) {
        aa->x[cd.mats[b]] = (const __nv_bfloat16*)(base + cd.off_x0 + b * (size_t)cd.kp * cd.lp * 2);
        aa->lp[cd.mats[b]] = cd.lp;
      }
    return launch(c, MUON_KIND_APPLY_X0,
                  [&] { launch_pdl(apply_x0_kernel, dim3(64, nm), dim3(256), 0, c.stream, *aa); });
  }

  int rc0 = update_wmaps(c, plan, gidx, io);
  if (rc0) return rc0;
  auto ga = std::make_unique<GemmArgs>();
  std::memset(ga.get(), 0, sizeof(GemmArgs));
  ga->tmaps = tmaps;
  ga->wmaps = (const CUtensorMap*)((char*)plan.tmaps + g.off_wmaps);
  ga->scale = scale;
  ga->status = c.status_d;
  ga->wait_limit_ns = g_wait_limit_ns;
  ga->nclasses = (int)g.classes.size();
  ga->a = io.a; ga->b = io.b; ga->c = io.c; ga->lr = io.lr;
  ga->assign = io.assign;
  fill_out(ga->out);
  // e4m3 operands only where the phases run as separate launches: in the
  // chained launch the extra e4m3 copies the epilogues write cost more than
  // the halved K-loops save (measured slower on every chained workload)
  const int fp8_iters = chain ? 0 : std::min(io.fp8_iters, io.ns_steps);
  if (fp8_iters > 0) {
    ga->tmaps8 = (const CUtensorMap*)((char*)plan.tmaps8 + g.off_tmaps8);
    ga->fp8_iters = fp8_iters;
    e4m3_scales(io.a, io.b, io.c, ga->sx8, ga->sa8);
  }

  if (chain) {
    ChainTables* ct = nullptr;
    int rc = get_chain(c, plan, gidx, io.ns_steps, &ct);
    if (rc) return rc;
    for (size_t ci = 0; ci < g.sym_cls.size(); ++ci) ga->cls[ci] = g.sym_cls[ci];
    ga->items = ct->items;
    ga->item_off = ct->off;
    ga->done = done;
    ga->debug_flags = 0;
    if (g_debug_flags & 1) { ga->debug_flags = 1; g_debug_flags &= ~1; }
    ga->final_apply = 1;                     // its items include the last update (W -= lr*O)
    return launch(c, MUON_KIND_CHAIN, [&] { launch_gemm(c.stream, *ga, c.sm_count, ct->nclusters); });
  }

  for (int it = 0; it < io.ns_steps; ++it) {
    for (int mode = kModeGram; mode <= kModeUpdate; ++mode) {
      const bool sym = mode != kModeUpdate;
      const auto& cls = sym ? g.sym_cls : g.upd_cls;
      for (size_t ci = 0; ci < cls.size(); ++ci) {
        ga->cls[ci] = cls[ci];
        if (mode == kModePoly) ga->cls[ci].kblocks = cls[ci].kp / kBK;
      }
      ga->total_tiles = sym ? g.sym_tiles : g.upd_tiles;
#ifdef MUON_DEBUG_BOUNDS
      // injection (debug bit 5): one tile index past the end for every cluster
      if (g_debug_flags & 32) { ga->total_tiles += std::max(1, c.sm_count / 2); g_debug_flags &= ~32; }
#endif
      ga->mode = mode;
      ga->x_in = it & 1;
      ga->first = it == 0;
      ga->iter = it;
      ga->final_apply = (mode == kModeUpdate) && (it == io.ns_steps - 1);
      ga->debug_flags = 0;
      if (g_debug_flags & 1) { ga->debug_flags = 1; g_debug_flags &= ~1; }
      const int kind = mode == kModeGram ? MUON_KIND_GRAM
                       : mode == kModePoly ? MUON_KIND_POLY
                       : (ga->final_apply ? MUON_KIND_UPDATE_APPLY : MUON_KIND_UPDATE);
      int rc = launch(c, kind, [&] { launch_gemm(c.stream, *ga, c.sm_count); });
      if (rc) return rc;
    }
  }
  return MUON_OK;
}

// Arguments of one fused launch (single-CTA or CTA-pair kernel) over
// mats[base, base + nm); lp is the padded long side each kernel works with.
std::unique_ptr<SmallArgs> fused_args(const std::vector<MatDesc>& mats, size_t base, int nm, const StepIO& io,
                                      int* status, bool pair) {
  auto sa = std::make_unique<SmallArgs>();
  std::memset(sa.get(), 0, sizeof(SmallArgs));
  sa->nmats = nm;
  sa->ns_steps = io.ns_steps;
  sa->nesterov = io.nesterov;
  sa->has_buf = io.buf != nullptr;
  sa->assign = io.assign;
  sa->mu = io.mu; sa->eps = io.eps; sa->a = io.a; sa->b = io.b; sa->c = io.c; sa->lr = io.lr;
  sa->status = status;
  sa->wait_limit_ns = g_wait_limit_ns;
  for (int i = 0; i < nm; ++i) {
    const MatDesc& d = mats[base + i];
    SmallMat& m = sa->mats[i];
    m.g = io.g[d.user];
    m.buf = io.buf ? io.buf[d.user] : nullptr;
    m.w = io.W[d.user];
    m.m = d.m; m.n = d.n; m.trans = d.trans;
    m.vec = (d.n % 4 == 0) && aligned16(m.g) && aligned16(m.w) && (!m.buf || aligned16(m.buf));
    m.lp = pair ? kPairMaxL : round_up(d.l, 64);
  }
  return sa;
}

// Runs `go` as launch kind `kind`: through the context's bookkeeping when
// there is one, else directly (the no-allocation entry point).
template <class F>
int launch_fused(Ctx* c, int kind, F&& go) {
  if (c) return launch(*c, kind, go);
  go();
  CUDA_TRY(cudaGetLastError());
  g_launches.fetch_add(1);
  return MUON_OK;
}

// One launch of the fused single-CTA kernel per kMaxMats small matrices (one CTA each).
int run_small(Ctx* c, cudaStream_t stream, const std::vector<MatDesc>& small, const StepIO& io, int* status) {
  for (size_t base = 0; base < small.size(); base += kMaxMats) {
    const int nm = (int)std::min<size_t>(kMaxMats, small.size() - base);
    auto sa = fused_args(small, base, nm, io, status, false);
    int rc = launch_fused(c, MUON_KIND_SMALL, [&] {
      launch_pdl(ns_small_kernel, dim3(nm), dim3(kSmallThreads), kSmallSmem, stream, *sa);
    });
    if (rc) return rc;
  }
  return MUON_OK;
}

// One launch of the fused CTA-pair kernel per kMaxMats matrices (one cluster of two CTAs each).
int run_pair(Ctx* c, cudaStream_t stream, const std::vector<MatDesc>& mats, const StepIO& io, int* status) {
  for (size_t base = 0; base < mats.size(); base += kMaxMats) {
    const int nm = (int)std::min<size_t>(kMaxMats, mats.size() - base);
    auto sa = fused_args(mats, base, nm, io, status, true);
    if (g_debug_flags & 2) { sa->debug_flags = 1; g_debug_flags &= ~2; }
    int rc = launch_fused(c, MUON_KIND_PAIR, [&] {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(2 * nm, 1, 1);
      cfg.blockDim = dim3(kPairThreads, 1, 1);
      cfg.dynamicSmemBytes = kPairSmem;
      cfg.stream = stream;
      cudaLaunchAttribute attr[2];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = 2;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
      attr[1].val.programmaticStreamSerializationAllowed = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 2;
      cudaLaunchKernelEx(&cfg, ns_pair_kernel, *sa);
    });
    if (rc) return rc;
  }
  return MUON_OK;
}

// One launch of the fused four-CTA kernel over every matrix routed to it (a cluster each).
int run_quad(Ctx* c, cudaStream_t stream, const std::vector<MatDesc>& mats, const StepIO& io, int* status) {
  const int nm = (int)mats.size();
  auto sa = fused_args(mats, 0, nm, io, status, false);
  if (g_debug_flags & 8) { sa->debug_flags = 1; g_debug_flags &= ~8; }
  return launch_fused(c, MUON_KIND_QUAD, [&] {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(4 * nm, 1, 1);
    cfg.blockDim = dim3(kQuadThreads, 1, 1);
    cfg.dynamicSmemBytes = kQuadSmem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 4;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    cudaLaunchKernelEx(&cfg, ns_quad_kernel, *sa);
  });
}

int validate_common(const int64_t* shapes, int n, int ns_steps) {
  if (!shapes) return fail(MUON_ERR_INVALID_ARG, "shapes is null");
  if (n <= 0) return fail(MUON_ERR_INVALID_ARG, "n must be > 0");
  if (ns_steps < 0 || ns_steps > 1000) return fail(MUON_ERR_INVALID_ARG, "ns_steps must be in [0, 1000]");
  for (int i = 0; i < 2 * n; ++i)
    if (shapes[i] <= 0) return fail(MUON_ERR_SHAPE, "shape entry " + std::to_string(i) + " is <= 0");
  return MUON_OK;
}

int validate_ptrs(const void* const* arr, int n, const char* what) {
  if (!arr) return fail(MUON_ERR_INVALID_ARG, std::string(what) + " array is null");
  for (int i = 0; i < n; ++i)
    if (!arr[i]) return fail(MUON_ERR_INVALID_ARG, std::string(what) + "[" + std::to_string(i) + "] is null");
  return MUON_OK;
}

int step_impl(const StepIO& io, const int64_t* shapes, int n, void* stream) {
  struct Range {                                     // one NVTX range per library call
    Range() { nvtxRangePushA("muon.step"); }
    ~Range() { nvtxRangePop(); }
  } range;
  Ctx* c = nullptr;
  int rc = get_ctx(stream, &c);
  if (rc) return rc;
  if ((rc = check_status(*c))) return rc;
  Plan* plan = nullptr;
  if ((rc = get_plan(*c, shapes, n, &plan, io.fp8_iters > 0 && io.ns_steps > 0))) return rc;
  if (!plan->small.empty() && (rc = run_small(c, c->stream, plan->small, io, c->status_d))) return rc;
  if (!plan->pair.empty() && (rc = run_pair(c, c->stream, plan->pair, io, c->status_d))) return rc;
  if (!plan->quad.empty() && (rc = run_quad(c, c->stream, plan->quad, io, c->status_d))) return rc;
  for (size_t gi = 0; gi < plan->groups.size(); ++gi)
    if ((rc = run_group(*c, *plan, gi, io))) return rc;
  return MUON_OK;
}

// One launch of o16_kernel per kMaxMats matrices: apply = 0 rounds src (fp32)
// into o16, apply = 1 adds -lr * o16 into w.
int run_o16(Ctx& c, int apply, float lr, const float* const* src, __nv_bfloat16* const* o16, float* const* w,
            const int64_t* shapes, int n) {
  for (int base = 0; base < n; base += kMaxMats) {
    const int nm = std::min(kMaxMats, n - base);
    auto oa = std::make_unique<O16Args>();
    std::memset(oa.get(), 0, sizeof(O16Args));
    oa->nmats = nm;
    oa->apply = apply;
    oa->lr = lr;
    long long most = 0;
    for (int i = 0; i < nm; ++i) {
      const int u = base + i;
      const long long cnt = (long long)shapes[2 * u] * shapes[2 * u + 1];
      oa->count[i] = cnt;
      oa->o16[i] = o16[u];
      if (apply) oa->w[i] = w[u]; else oa->src[i] = src[u];
      oa->vec[i] = cnt % 8 == 0 && aligned16(o16[u]) && aligned16(apply ? (const void*)w[u] : (const void*)src[u]);
      most = std::max(most, cnt);
    }
    // about 8 elements per thread per pass, and some 1200 CTAs over the launch
    const long long want = (most + 2047) / 2048;
    const int gx = (int)std::max<long long>(1, std::min<long long>(want, std::max(4, 1184 / nm)));
    int rc = launch(c, MUON_KIND_O16,
                    [&] { launch_pdl(o16_kernel, dim3(gx, nm), dim3(256), 0, c.stream, *oa); });
    if (rc) return rc;
  }
  return MUON_OK;
}

}  // namespace

// =================================================================== C ABI ===
extern "C" {

int muon_update_bf16(const float* const* grads, float* const* momentum_bufs, uint16_t* const* O, const int64_t* shapes,
                     int n, float mu, int ns_steps, float a, float b, float c, float eps, int nesterov, void* stream) {
  std::lock_guard<std::mutex> lk(g_mu);
  int rc = validate_common(shapes, n, ns_steps);
  if (rc) return rc;
  if ((rc = validate_ptrs((const void* const*)grads, n, "grads"))) return rc;
  if ((rc = validate_ptrs((const void* const*)momentum_bufs, n, "momentum_bufs"))) return rc;
  if ((rc = validate_ptrs((const void* const*)O, n, "O"))) return rc;
  if (nesterov != 0 && nesterov != 1) return fail(MUON_ERR_INVALID_ARG, "nesterov must be 0 or 1");
  if (!(eps >= 0.f)) return fail(MUON_ERR_INVALID_ARG, "eps must be >= 0");
  Ctx* ctx = nullptr;
  if ((rc = get_ctx(stream, &ctx))) return rc;
  std::vector<size_t> off(n);
  size_t total = 0;
  for (int i = 0; i < n; ++i) {
    off[i] = total;
    total += align_up((size_t)(shapes[2 * i] * shapes[2 * i + 1]), 64);
  }
  if (ctx->o32_cap < total) {
    CUDA_TRY(cudaStreamSynchronize(ctx->stream));
    if (ctx->o32) cudaFree(ctx->o32);
    ctx->o32 = nullptr;
    ctx->o32_cap = 0;
    if (cudaMalloc((void**)&ctx->o32, total * sizeof(float)) != cudaSuccess) {
      cudaGetLastError();
      return fail(MUON_ERR_NOMEM, "fp32 update scratch allocation failed");
    }
    ctx->o32_cap = total;
  }
  std::vector<float*> o32(n);
  for (int i = 0; i < n; ++i) o32[i] = ctx->o32 + off[i];
  // the step in assign mode writes O (fp32) where it would update W
  StepIO io{o32.data(), grads, momentum_bufs, 0.f, mu, a, b, c, eps, ns_steps, nesterov, 1};
  if ((rc = step_impl(io, shapes, n, stream))) return rc;
  return run_o16(*ctx, 0, 0.f, o32.data(), (__nv_bfloat16* const*)O, nullptr, shapes, n);
}

int muon_apply_bf16(float* const* params, const uint16_t* const* O, const int64_t* shapes, int n, float lr,
                    void* stream) {
  std::lock_guard<std::mutex> lk(g_mu);
  int rc = validate_common(shapes, n, 0);
  if (rc) return rc;
  if ((rc = validate_ptrs((const void* const*)params, n, "params"))) return rc;
  if ((rc = validate_ptrs((const void* const*)O, n, "O"))) return rc;
  Ctx* ctx = nullptr;
  if ((rc = get_ctx(stream, &ctx))) return rc;
  if ((rc = check_status(*ctx))) return rc;
  return run_o16(*ctx, 1, lr, nullptr, (__nv_bfloat16* const*)O, params, shapes, n);
}

int muon_step_ex(float* const* params, const float* const* grads, float* const* momentum_bufs,
                 const int64_t* shapes, int n, float lr, float mu, int ns_steps,
                 float a, float b, float c, float eps, int nesterov, void* stream) {
  std::lock_guard<std::mutex> lk(g_mu);
  int rc = validate_common(shapes, n, ns_steps);
  if (rc) return rc;
  if ((rc = validate_ptrs((const void* const*)params, n, "params"))) return rc;
  if ((rc = validate_ptrs((const void* const*)grads, n, "grads"))) return rc;
  if ((rc = validate_ptrs((const void* const*)momentum_bufs, n, "momentum_bufs"))) return rc;
  if (nesterov != 0 && nesterov != 1) return fail(MUON_ERR_INVALID_ARG, "nesterov must be 0 or 1");
  if (!(eps >= 0.f)) return fail(MUON_ERR_INVALID_ARG, "eps must be >= 0");
  StepIO io{params, grads, momentum_bufs, lr, mu, a, b, c, eps, ns_steps, nesterov, 0};
  return step_impl(io, shapes, n, stream);
}

int muon_step_fp8(float* const* params, const float* const* grads, float* const* momentum_bufs,
                  const int64_t* shapes, int n, float lr, float mu, int ns_steps, float a, float b, float c,
                  float eps, int nesterov, int fp8_iters, void* stream) {
  std::lock_guard<std::mutex> lk(g_mu);
  int rc = validate_common(shapes, n, ns_steps);
  if (rc) return rc;
  if ((rc = validate_ptrs((const void* const*)params, n, "params"))) return rc;
  if ((rc = validate_ptrs((const void* const*)grads, n, "grads"))) return rc;
  if ((rc = validate_ptrs((const void* const*)momentum_bufs, n, "momentum_bufs"))) return rc;
  if (nesterov != 0 && nesterov != 1) return fail(MUON_ERR_INVALID_ARG, "nesterov must be 0 or 1");
  if (!(eps >= 0.f)) return fail(MUON_ERR_INVALID_ARG, "eps must be >= 0");
  if (fp8_iters < 0 || fp8_iters > kMaxFp8Iters)
    return fail(MUON_ERR_INVALID_ARG, "fp8_iters must be in [0, " + std::to_string(kMaxFp8Iters) + "]");
  StepIO io{params, grads, momentum_bufs, lr, mu, a, b, c, eps, ns_steps, nesterov, 0, fp8_iters};
  return step_impl(io, shapes, n, stream);
}

int muon_step(float* const* params, const float* const* grads, float* const* momentum_bufs,
              const int64_t* shapes, int n, float lr, float mu, int ns_steps, void* stream) {
  return muon_step_ex(params, grads, momentum_bufs, shapes, n, lr, mu, ns_steps, MUON_NS_A, MUON_NS_B, MUON_NS_C,
                      MUON_NS_EPS, 1, stream);
}

int muon_orthogonalize(const float* const* G, float* const* O, const int64_t* shapes, int n, int ns_steps,
                       void* stream) {
  std::lock_guard<std::mutex> lk(g_mu);
  int rc = validate_common(shapes, n, ns_steps);
  if (rc) return rc;
  if ((rc = validate_ptrs((const void* const*)G, n, "G"))) return rc;
  if ((rc = validate_ptrs((const void* const*)O, n, "O"))) return rc;
  StepIO io{O, G, nullptr, 0.f, 0.f, MUON_NS_A, MUON_NS_B, MUON_NS_C, MUON_NS_EPS, ns_steps, 1, 1};
  return step_impl(io, shapes, n, stream);
}

int muon_step_host(float* const* params, const float* const* grads, float* const* momentum_bufs,
                   const int64_t* shapes, int n, float lr, float mu, int ns_steps, void* stream) {
  std::lock_guard<std::mutex> lk(g_mu);
  int rc = validate_common(shapes, n, ns_steps);
  if (rc) return rc;
  if ((rc = validate_ptrs((const void* const*)params, n, "params"))) return rc;
  if ((rc = validate_ptrs((const void* const*)grads, n, "grads"))) return rc;
  if ((rc = validate_ptrs((const void* const*)momentum_bufs, n, "momentum_bufs"))) return rc;
  Ctx* c = nullptr;
  if ((rc = get_ctx(stream, &c))) return rc;
  if ((rc = check_status(*c))) return rc;
  size_t total = 0;
  for (int i = 0; i < n; ++i) total += align_up((size_t)(shapes[2 * i] * shapes[2 * i + 1]), 64);
  const size_t need = 3 * total * sizeof(float);
  if (c->stage_cap < need) {
    CUDA_TRY(cudaStreamSynchronize(c->stream));
    if (c->stage) cudaFree(c->stage);
    c->stage = nullptr;
    c->stage_cap = 0;
    if (cudaMalloc((void**)&c->stage, need) != cudaSuccess) {
      cudaGetLastError();
      return fail(MUON_ERR_NOMEM, "staging allocation failed");
    }
    c->stage_cap = need;
  }
  if (!c->h2d) CUDA_TRY(cudaStreamCreateWithFlags(&c->h2d, cudaStreamNonBlocking));
  if (!c->d2h) CUDA_TRY(cudaStreamCreateWithFlags(&c->d2h, cudaStreamNonBlocking));
  std::vector<float*> dW(n), dg(n), db(n);
  {
    size_t off = 0;
    for (int i = 0; i < n; ++i) {
      dW[i] = c->stage + off;
      dg[i] = c->stage + total + off;
      db[i] = c->stage + 2 * total + off;
      off += align_up((size_t)(shapes[2 * i] * shapes[2 * i + 1]), 64);
    }
  }
  // Chunks of consecutive matrices: copies in (stream h2d), the step (caller's
  // stream) and copies out (stream d2h) of different chunks overlap.
  const size_t chunk_bytes = std::max<size_t>(size_t(32) << 20, need / 16);
  std::vector<std::pair<int, int>> chunks;
  for (int i = 0; i < n;) {
    int j = i;
    size_t bytes = 0;
    while (j < n && (j == i || bytes + 12 * (size_t)(shapes[2 * j] * shapes[2 * j + 1]) <= chunk_bytes)) {
      bytes += 12 * (size_t)(shapes[2 * j] * shapes[2 * j + 1]);
      ++j;
    }
    chunks.push_back({i, j});
    i = j;
  }
  while (c->host_events.size() < 2 * chunks.size()) {
    cudaEvent_t e;
    CUDA_TRY(cudaEventCreateWithFlags(&e, cudaEventDisableTiming));
    c->host_events.push_back(e);
  }
  // the step of a chunk must not start before earlier work on the caller's stream
  cudaEvent_t* ev = c->host_events.data();
  CUDA_TRY(cudaEventRecord(ev[0], c->stream));
  CUDA_TRY(cudaStreamWaitEvent(c->h2d, ev[0], 0));
  for (size_t ci = 0; ci < chunks.size(); ++ci) {
    const int i0 = chunks[ci].first, i1 = chunks[ci].second;
    for (int i = i0; i < i1; ++i) {
      const size_t e = (size_t)(shapes[2 * i] * shapes[2 * i + 1]);
      CUDA_TRY(cudaMemcpyAsync(dW[i], params[i], e * 4, cudaMemcpyHostToDevice, c->h2d));
      CUDA_TRY(cudaMemcpyAsync(dg[i], grads[i], e * 4, cudaMemcpyHostToDevice, c->h2d));
      CUDA_TRY(cudaMemcpyAsync(db[i], momentum_bufs[i], e * 4, cudaMemcpyHostToDevice, c->h2d));
    }
    CUDA_TRY(cudaEventRecord(ev[2 * ci], c->h2d));
    CUDA_TRY(cudaStreamWaitEvent(c->stream, ev[2 * ci], 0));
    Plan* plan = nullptr;
    if ((rc = get_plan(*c, shapes + 2 * i0, i1 - i0, &plan))) return rc;
    // StepIO indexes by the caller's matrix index within this chunk
    StepIO io{dW.data() + i0, (const float* const*)dg.data() + i0, db.data() + i0, lr, mu, MUON_NS_A, MUON_NS_B,
              MUON_NS_C, MUON_NS_EPS, ns_steps, 1, 0};
    if (!plan->small.empty() && (rc = run_small(c, c->stream, plan->small, io, c->status_d))) return rc;
    if (!plan->pair.empty() && (rc = run_pair(c, c->stream, plan->pair, io, c->status_d))) return rc;
    if (!plan->quad.empty() && (rc = run_quad(c, c->stream, plan->quad, io, c->status_d))) return rc;
    for (size_t gi = 0; gi < plan->groups.size(); ++gi)
      if ((rc = run_group(*c, *plan, gi, io))) return rc;
    CUDA_TRY(cudaEventRecord(ev[2 * ci + 1], c->stream));
    CUDA_TRY(cudaStreamWaitEvent(c->d2h, ev[2 * ci + 1], 0));
    for (int i = i0; i < i1; ++i) {
      const size_t e = (size_t)(shapes[2 * i] * shapes[2 * i + 1]);
      CUDA_TRY(cudaMemcpyAsync(params[i], dW[i], e * 4, cudaMemcpyDeviceToHost, c->d2h));
      CUDA_TRY(cudaMemcpyAsync(momentum_bufs[i], db[i], e * 4, cudaMemcpyDeviceToHost, c->d2h));
    }
  }
  CUDA_TRY(cudaStreamSynchronize(c->d2h));
  CUDA_TRY(cudaStreamSynchronize(c->stream));
  return check_status(*c);
}

int muon_guard_check(void* stream) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (!guard_bands()) return fail(MUON_ERR_UNSUPPORTED, "guard bands are off (MUON_GUARD_BANDS=1 when loading)");
  Ctx* c = nullptr;
  int rc = get_ctx(stream, &c);
  if (rc) return rc;
  CUDA_TRY(cudaStreamSynchronize(c->stream));
  std::vector<unsigned char> h(kGuardBytes);
  long long changed = 0;
  for (size_t off : c->guards) {
    CUDA_TRY(cudaMemcpy(h.data(), (char*)c->ws + off, kGuardBytes, cudaMemcpyDeviceToHost));
    for (unsigned char v : h) changed += v != kGuardByte;
  }
  return (int)std::min<long long>(changed, 0x7fffffff);
}

size_t muon_workspace_size(const int64_t* shapes, int n) {
  if (!shapes || n <= 0) return 0;
  for (int i = 0; i < 2 * n; ++i)
    if (shapes[i] <= 0) return 0;
  Plan p;
  if (build_layout(shapes, n, p)) return 0;
  return std::max<size_t>(p.ws_bytes, kTicketBytes);
}

int muon_sync_status(void* stream) {
  std::lock_guard<std::mutex> lk(g_mu);
  Ctx* c = nullptr;
  int rc = get_ctx(stream, &c);
  if (rc) return rc;
  CUDA_TRY(cudaStreamSynchronize(c->stream));
  return check_status(*c);
}

const char* muon_last_error(void) { return g_last_error.c_str(); }

void muon_release(void) {
  std::lock_guard<std::mutex> lk(g_mu);
  int cur = 0;
  cudaGetDevice(&cur);
  for (auto& kv : g_ctx) {
    Ctx& c = *kv.second;
    cudaSetDevice(c.dev);
    cudaStreamSynchronize(c.stream);
    if (c.ws) cudaFree(c.ws);
    if (c.stage) cudaFree(c.stage);
    if (c.o32) cudaFree(c.o32);
    if (c.status_h) cudaFreeHost(c.status_h);
    for (auto& r : c.prof) { cudaEventDestroy(r.a); cudaEventDestroy(r.b); }
    for (auto e : c.event_pool) cudaEventDestroy(e);
    for (auto e : c.host_events) cudaEventDestroy(e);
    if (c.h2d) cudaStreamDestroy(c.h2d);
    if (c.d2h) cudaStreamDestroy(c.d2h);
  }
  g_ctx.clear();
  g_dev_ready.clear();                     // a context created after this is set up again
  cudaSetDevice(cur);
}

int muon_profile_enable(int enable) {
  std::lock_guard<std::mutex> lk(g_mu);
  g_profile = enable != 0;
  return MUON_OK;
}

int muon_profile_read(double* ms, int64_t* launches, int nkinds) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (!ms || !launches || nkinds <= 0) return fail(MUON_ERR_INVALID_ARG, "bad profile buffers");
  for (auto& kv : g_ctx) {
    Ctx& c = *kv.second;
    for (auto& r : c.prof) {
      if (cudaEventSynchronize(r.b) != cudaSuccess) return fail(MUON_ERR_CUDA, "event synchronize failed");
      float t = 0.f;
      cudaEventElapsedTime(&t, r.a, r.b);
      if (r.kind < nkinds) { ms[r.kind] += t; launches[r.kind] += 1; }
      c.event_pool.push_back(r.a);
      c.event_pool.push_back(r.b);
    }
    c.prof.clear();
  }
  return MUON_OK;
}

int64_t muon_launch_count(void) { return g_launches.load(); }

int muon_chain_clusters(void) {
  std::lock_guard<std::mutex> lk(g_mu);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || device_setup(dev) != MUON_OK) {
    cudaGetLastError();
    return -1;
  }
  return g_chain_clusters[dev];
}

int muon_chain_plan(const int64_t* shapes, int n, int ns_steps, int nclusters, int32_t* items, int64_t capacity,
                    int32_t* cluster_off, int64_t* nitems) {
  std::lock_guard<std::mutex> lk(g_mu);
  int rc = validate_common(shapes, n, ns_steps);
  if (rc) return rc;
  if (!nitems || !cluster_off || nclusters < 1 || nclusters > 4096)
    return fail(MUON_ERR_INVALID_ARG, "nitems and cluster_off must be given, 1 <= nclusters <= 4096");
  Plan plan;
  if ((rc = build_layout(shapes, n, plan))) return rc;
  *nitems = 0;
  if (plan.groups.empty() || ns_steps < 1) {
    for (int c = 0; c <= nclusters; ++c) cluster_off[c] = 0;
    return MUON_OK;
  }
  std::vector<WorkItem> list;
  std::vector<int> off;
  build_chain(plan.groups[0], ns_steps, nclusters, list, off);
  *nitems = (int64_t)list.size();
  for (int c = 0; c <= nclusters; ++c) cluster_off[c] = off[c];
  if (!items || capacity < (int64_t)list.size())
    return fail(MUON_ERR_INVALID_ARG, "items holds fewer than " + std::to_string(list.size()) + " entries");
  const Group& g = plan.groups[0];
  for (size_t i = 0; i < list.size(); ++i) {
    const WorkItem& w = list[i];
    int32_t* o = items + 8 * i;
    o[0] = w.need; o[1] = g.mats[w.mat].user; o[2] = w.cls; o[3] = w.b;
    o[4] = w.tm; o[5] = w.tn; o[6] = w.mode; o[7] = w.it;
  }
  return MUON_OK;
}

int muon_debug_set(int flags, int64_t wait_limit_ns) {
  std::lock_guard<std::mutex> lk(g_mu);
  g_debug_flags = flags;
  g_wait_limit_ns = wait_limit_ns > 0 ? (uint64_t)wait_limit_ns : 2000000000ull;
  return MUON_OK;
}

}  // extern "C"

// ======================================================= no-allocation step ===
// muon_step_noalloc: the same Muon step for callers that must not allocate
// device memory -- for example code running inside a custom allocator or a
// memory-pool callback, or a host whose device memory is budgeted up front so
// that any cudaMalloc could fail or deadlock.  Its scratch (bf16 iterates,
// Gram / polynomial matrices, norm partials, scales, tensor-map table and a
// status word) lives in one file-scope device array of fixed size that every
// GPU loading this library holds until the process exits.
namespace {

constexpr size_t kNoAllocBytes = size_t(64) << 20;      // 64 MiB of static scratch per device
constexpr size_t kNoAllocTableBytes = size_t(64) << 10; // tensor maps + status word at the end

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocBytes];

// Device address of g_noalloc_scratch on the current device.  Host code only
// holds a host-side stand-in under that name, so the address is looked up
// with the device current -- on every call: once the module is loaded the
// lookup allocates nothing, and a fresh lookup stays right if the context was
// torn down and the module loaded again (the array's address can change).
int noalloc_scratch_address(void** out) {
  void* p = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
  if (e != cudaSuccess || !p)
    return fail(MUON_ERR_CUDA, std::string("cudaGetSymbolAddress(static scratch): ") + cudaGetErrorString(e));
  *out = p;
  return MUON_OK;
}

int noalloc_launch(cudaStream_t stream, char* base, const Plan& plan, const StepIO& io, int sm_count) {
  const Group& g = plan.groups[0];
  const size_t table_off = kNoAllocBytes - kNoAllocTableBytes;
  int* status = (int*)(base + kNoAllocBytes - 256);
  CUtensorMap* tmaps = (CUtensorMap*)(base + table_off);
  CUtensorMap* wmaps = tmaps + g.classes.size() * kTmapsPerClass;
  float* scale = (float*)(base + g.off_scale);
  const int nm = (int)g.mats.size();

  // The norm arrival counters must start at zero (the status word was read
  // and found clear at the start of the call).
  CUDA_TRY(cudaMemsetAsync(base, 0, kTicketBytes, stream));

  // Tensor maps of this call (scratch buffers and the caller's outputs), copied
  // from host memory into the table at the end of the scratch.
  std::vector<CUtensorMap> host(g.classes.size() * kTmapsPerClass + g.mats.size());
  std::memset(host.data(), 0, host.size() * sizeof(CUtensorMap));
  int rc;
  for (size_t ci = 0; ci < g.classes.size(); ++ci) {
    if ((rc = encode_class_maps(&host[ci * kTmapsPerClass], base, g.classes[ci]))) return rc;
  }
  CUtensorMap* hw = &host[g.classes.size() * kTmapsPerClass];
  for (size_t i = 0; i < g.mats.size(); ++i) {
    const MatDesc& d = g.mats[i];
    if (d.n % 4 == 0 && aligned16(io.W[d.user]))
      if ((rc = encode_wmap(&hw[i], (void*)io.W[d.user], d.m, d.n, d.trans))) return rc;
  }
  CUDA_TRY(cudaMemcpyAsync(tmaps, host.data(), host.size() * sizeof(CUtensorMap), cudaMemcpyHostToDevice, stream));

  // prologue: momentum, norm partials, bf16 iterate
  auto pa = std::make_unique<ProArgs>();
  std::memset(pa.get(), 0, sizeof(ProArgs));
  pa->nmats = nm;
  pa->total_tiles = g.pro_tiles;
  pa->mu = io.mu;
  pa->eps = io.eps;
  pa->nesterov = io.nesterov;
  pa->has_buf = 1;
  pa->partials = (float*)(base + g.off_partials);
  pa->tickets = (unsigned*)(base + g.off_tickets);
  pa->scale = scale;
  auto ga = std::make_unique<GemmArgs>();
  std::memset(ga.get(), 0, sizeof(GemmArgs));
  auto aa = std::make_unique<ApplyArgs>();
  std::memset(aa.get(), 0, sizeof(ApplyArgs));
  for (const auto& cd : g.classes)
    for (size_t b = 0; b < cd.mats.size(); ++b) {
      const int gi = cd.mats[b];
      const MatDesc& d = g.mats[gi];
      ProMat& pm = pa->mats[gi];
      pm.g = io.g[d.user];
      pm.buf = io.buf[d.user];
      pm.x = (__nv_bfloat16*)(base + cd.off_x0 + b * (size_t)cd.kp * cd.lp * 2);
      pm.m = d.m; pm.n = d.n; pm.kp = d.kp; pm.lp = d.lp;
      pm.trans = d.trans;
      pm.vec = (d.n % 4 == 0) && aligned16(pm.g) && aligned16(pm.buf);
      pm.tile_begin = g.pro_tile_begin[gi];
      pm.tiles_c = d.lp / kProCols;
      pm.tiles = (d.kp / kProRows) * pm.tiles_c;
      OutMat o;
      o.w = io.W[d.user];
      o.m = d.m; o.n = d.n; o.trans = d.trans;
      o.vec = (d.n % 4 == 0) && aligned16(o.w);
      o.tma = o.vec;
      ga->out[gi] = o;
      aa->out[gi] = o;
      aa->x[gi] = pm.x;
      aa->lp[gi] = cd.lp;
    }
  CUDA_TRY(launch_pdl(prologue_kernel, dim3(g.pro_tiles), dim3(kProThreads), 0, stream, *pa));
  g_launches.fetch_add(1);

  if (io.ns_steps == 0) {
    aa->scale = scale;
    aa->lr = io.lr;
    aa->assign = 0;
    aa->nmats = nm;
    CUDA_TRY(launch_pdl(apply_x0_kernel, dim3(64, nm), dim3(256), 0, stream, *aa));
    g_launches.fetch_add(1);
    return MUON_OK;
  }
  ga->tmaps = tmaps;
  ga->wmaps = wmaps;
  ga->scale = scale;
  ga->status = status;
  ga->wait_limit_ns = g_wait_limit_ns;
  ga->nclasses = (int)g.classes.size();
  ga->a = io.a; ga->b = io.b; ga->c = io.c; ga->lr = io.lr;
  ga->assign = 0;
  for (int it = 0; it < io.ns_steps; ++it) {
    for (int mode = kModeGram; mode <= kModeUpdate; ++mode) {
      const bool sym = mode != kModeUpdate;
      const auto& cls = sym ? g.sym_cls : g.upd_cls;
      for (size_t ci = 0; ci < cls.size(); ++ci) {
        ga->cls[ci] = cls[ci];
        if (mode == kModePoly) ga->cls[ci].kblocks = cls[ci].kp / kBK;
      }
      ga->total_tiles = sym ? g.sym_tiles : g.upd_tiles;
      ga->mode = mode;
      ga->x_in = it & 1;
      ga->first = it == 0;
      ga->final_apply = (mode == kModeUpdate) && (it == io.ns_steps - 1);
      ga->debug_flags = 0;
      if (g_debug_flags & 1) { ga->debug_flags = 1; g_debug_flags &= ~1; }
      CUDA_TRY(launch_gemm(stream, *ga, sm_count));
      g_launches.fetch_add(1);
    }
  }
  return MUON_OK;
}

}  // namespace

extern "C" int muon_step_noalloc(float* const* params, const float* const* grads, float* const* momentum_bufs,
                                 const int64_t* shapes, int n, float lr, float mu, int ns_steps, void* stream) {
  std::lock_guard<std::mutex> lk(g_mu);
  int rc = validate_common(shapes, n, ns_steps);
  if (rc) return rc;
  if ((rc = validate_ptrs((const void* const*)params, n, "params"))) return rc;
  if ((rc = validate_ptrs((const void* const*)grads, n, "grads"))) return rc;
  if ((rc = validate_ptrs((const void* const*)momentum_bufs, n, "momentum_bufs"))) return rc;
  Plan plan;
  if ((rc = build_layout(shapes, n, plan))) return rc;
  if (plan.groups.size() > 1)
    return fail(MUON_ERR_UNSUPPORTED, "muon_step_noalloc takes at most " + std::to_string(kMaxMats) +
                                          " matrices of at most " + std::to_string(kMaxClasses) +
                                          " padded shapes per call");
  const size_t table = plan.groups.empty() ? 0
                       : (plan.groups[0].classes.size() * kTmapsPerClass + plan.groups[0].mats.size()) *
                             sizeof(CUtensorMap);
  if (plan.ws_bytes > kNoAllocBytes - kNoAllocTableBytes || table > kNoAllocTableBytes - 256)
    return fail(MUON_ERR_UNSUPPORTED, "muon_step_noalloc: these shapes need " + std::to_string(plan.ws_bytes) +
                                          " bytes of scratch; the static scratch holds " +
                                          std::to_string(kNoAllocBytes - kNoAllocTableBytes) +
                                          " (split the matrices over several calls)");
  int dev = 0;
  CUDA_TRY(cudaGetDevice(&dev));
  if ((rc = device_setup(dev))) return rc;
  void* base = nullptr;
  if ((rc = noalloc_scratch_address(&base))) return rc;
  int sm_count = 148;
  CUDA_TRY(cudaDeviceGetAttribute(&sm_count, cudaDevAttrMultiProcessorCount, dev));
  StepIO io{params, grads, momentum_bufs, lr, mu, MUON_NS_A, MUON_NS_B, MUON_NS_C, MUON_NS_EPS, ns_steps, 1, 0};
  // The status word at the end of the scratch holds what the kernels of the
  // previous call on this device recorded: wait for that call, report a
  // bounded wait that ran out (and clear the word), else go on with it clear.
  int* status = (int*)((char*)base + kNoAllocBytes - 256);
  int prev = 0;
  CUDA_TRY(cudaMemcpyAsync(&prev, status, sizeof(int), cudaMemcpyDeviceToHost, (cudaStream_t)stream));
  CUDA_TRY(cudaStreamSynchronize((cudaStream_t)stream));
  if (prev != 0) {
    CUDA_TRY(cudaMemsetAsync(status, 0, sizeof(int), (cudaStream_t)stream));
    CUDA_TRY(cudaStreamSynchronize((cudaStream_t)stream));
    return status_error(prev, "an earlier muon_step_noalloc call (nothing was launched by this one)");
  }
  if (!plan.small.empty() && (rc = run_small(nullptr, (cudaStream_t)stream, plan.small, io, status))) return rc;
  if (!plan.pair.empty() && (rc = run_pair(nullptr, (cudaStream_t)stream, plan.pair, io, status))) return rc;
  if (!plan.quad.empty() && (rc = run_quad(nullptr, (cudaStream_t)stream, plan.quad, io, status))) return rc;
  if (plan.groups.empty()) return MUON_OK;
  return noalloc_launch((cudaStream_t)stream, (char*)base, plan, io, sm_count);
}
