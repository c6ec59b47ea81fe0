// muon_api.cu -- the C interface declared in include/muon.h.
//
// Host side only: argument checks, the per-device plan cache (scratch
// buffers, TMA tensor maps, tile lists, work queues) and the launch sequence
//
//   K1 (momentum + norm + cast)  ->  [GRAM -> POLY -> UPDATE] x ns_steps
//
// where the last UPDATE applies the parameter update in its epilogue.  All
// matrices of a call share each launch (grouped by phase), so the many small
// GPT-2 matrices fill the GPU together.
#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <map>
#include <memory>
#include <mutex>
#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "internal.h"
#ifdef MUON_BOUNDS_CHECK
#include "muon_debug.h"
#endif

namespace muon {
namespace {

constexpr float kDefaultCoeffs[3] = {3.4445f, -4.7750f, 2.0315f};
constexpr int kMaxSteps = 100;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

std::mutex g_mutex;
unsigned long long g_limit_ns = 2000000000ull;
bool g_limit_from_env = false;

long long round_up(long long v, long long m) { return (v + m - 1) / m * m; }
long long cdiv(long long a, long long b) { return (a + b - 1) / b; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 2-D bf16 tensor map: rows x cols, row pitch ld elements, 64x64 boxes,
// 128-byte swizzle, zero fill outside the tensor.
bool make_map(CUtensorMap* map, const void* base, long long rows, long long cols, long long ld) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(ld * 2)};
  cuuint32_t box[2] = {(cuuint32_t)BOX, (cuuint32_t)BOX};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Output map for TMA stores, in the layout of the epilogue's staging blocks:
// 32 x 32 bf16 boxes with 64-byte swizzle (symmetric outputs, which also
// store each block mirrored), or 32 rows x 64 columns with 128-byte swizzle
// (X-update outputs: two chunks per store).
bool make_out_map(CUtensorMap* map, const void* base, long long rows, long long cols, long long ld,
                  bool wide = false) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(ld * 2)};
  cuuint32_t box[2] = {(cuuint32_t)(wide ? 2 * OUT_BOX : OUT_BOX), (cuuint32_t)OUT_BOX};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   wide ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// fp32 parameter map for the last X update: 32 x 32 boxes, 128-byte swizzle.
// Needs the row pitch (cols * 4 bytes) to be a multiple of 16 bytes.
bool make_param_map(CUtensorMap* map, const void* base, long long rows, long long cols) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(cols * 4)};
  cuuint32_t box[2] = {32, 32};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// ---------------------------------------------------------------- device memory arena

// Guard bands: every region a plan hands out is followed by kGuardBytes of
// a fixed byte pattern, written when the plan is built and never touched by
// any kernel.  muon_guard_check() reads them back: a changed byte means some
// kernel wrote past the end of a region.
constexpr size_t kGuardBytes = 256;
constexpr unsigned char kGuardByte = 0xA5;

struct Arena {
  size_t off = 0;
  std::vector<size_t> guards;   // offsets of the guard bands
  size_t take(size_t bytes, size_t align = 256) {
    off = (off + align - 1) / align * align;
    size_t at = off;
    off += bytes;
    off = (off + 255) / 256 * 256;
    guards.push_back(off);
    off += kGuardBytes;
    return at;
  }
};

struct DevBlock {
  char* ptr = nullptr;
  size_t bytes = 0;
  ~DevBlock() {
    if (ptr) cudaFree(ptr);
  }
};

// ---------------------------------------------------------------- plans

struct Geom {
  long long r, c, m, n, ldx, lda;
  int transposed;
};

struct NsPhase {
  NsProblem* probs = nullptr;  // device
  NsTile* tiles = nullptr;     // device
  int ntiles = 0;
};

struct K1Plan {
  K1Info* info = nullptr;
  K1Item* items = nullptr;
  int nitems = 0;
  int* counters = nullptr;  // [1 + 2n]: head, done[n], ready[n]; then the chain's deps
  double* partials = nullptr;
  double* norms = nullptr;
  int n = 0;
  int npartials = 0;
};

struct Plan {
  std::vector<Geom> geom;
  DevBlock mem;
  __nv_bfloat16* X[2] = {nullptr, nullptr};  // ping-pong iterates (base of all matrices)
  std::vector<long long> x_off, a_off;       // per-matrix offsets (elements)
  __nv_bfloat16* A = nullptr;
  __nv_bfloat16* B = nullptr;
  NsPhase gram[2], poly, upd[2];
  K1Plan k1;
  std::vector<size_t> guards;                // guard band offsets in mem
  // Chain tile lists (device), one per number of iterations used so far.
  struct Chain {
    std::unique_ptr<DevBlock> mem;
    int ntiles = 0;
  };
  std::map<int, Chain> chains;
  int* deps = nullptr;                       // 3 kMaxSteps n chain counters
  // Parameter tensor maps of the last X update, one device block per set of
  // parameter pointers, most recently used first (at most kParamMapSets).
  struct ParamMaps {
    std::vector<const void*> ptrs;
    std::unique_ptr<DevBlock> mem;
  };
  std::vector<ParamMaps> pmaps;
  // Device table of mirror destinations of the last X update, valid for the
  // host pointers in mirror_for (rebuilt when a call passes others).
  DevBlock mirror_mem;
  std::vector<const void*> mirror_for;
};

struct DeviceCtx {
  int device = -1;
  int num_sms = 0;
  int k1_blocks_per_sm = 1;
  int adamw_blocks_per_sm = 1;
  int max_pairs = 1;           // co-resident CTA pairs of the GEMM kernels
  int* status = nullptr;
  std::map<std::vector<long long>, std::unique_ptr<Plan>> plans;
  std::map<std::vector<long long>, std::unique_ptr<Plan>> stage_plans;
};

std::map<int, std::unique_ptr<DeviceCtx>> g_ctx;

// ---------------------------------------------------------------- profiling events
enum ProfKind : int {
  PK_K1 = 0, PK_GRAM = 1, PK_POLY = 2, PK_UPDATE = 3, PK_FINAL = 4, PK_APPLY = 5, PK_ADAMW = 6,
  PK_CHAIN = 7
};

struct ProfRecord {
  int kind;
  cudaEvent_t start, stop;
};

struct Profiler {
  bool on = false;
  std::vector<ProfRecord> recs;
  std::vector<cudaEvent_t> pool;
  cudaEvent_t get() {
    if (!pool.empty()) {
      cudaEvent_t e = pool.back();
      pool.pop_back();
      return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
  }
};

Profiler g_prof;

// Records an event pair around one launch when profiling is on.
// Names of the launch kinds, for NVTX ranges (a profiler's timeline shows
// each launch of this library under its name; without a profiler attached
// an NVTX range costs a few nanoseconds of host time).
const char* const kProfNames[] = {"muon: momentum/norm/cast", "muon: Gram",
                                  "muon: polynomial",         "muon: X update",
                                  "muon: final X update",     "muon: update (no NS)",
                                  "muon: AdamW",              "muon: NS chain"};

struct ProfScope {
  int kind;
  cudaStream_t stream;
  cudaEvent_t start = nullptr;
  ProfScope(int k, cudaStream_t s) : kind(k), stream(s) {
    nvtxRangePushA(kProfNames[k]);
    if (g_prof.on) {
      start = g_prof.get();
      if (start) cudaEventRecord(start, stream);
    }
  }
  ~ProfScope() {
    nvtxRangePop();
    if (!start) return;
    cudaEvent_t stop = g_prof.get();
    if (!stop) return;
    cudaEventRecord(stop, stream);
    g_prof.recs.push_back({kind, start, stop});
  }
};

int cuda_err(cudaError_t e) { return e == cudaSuccess ? MUON_OK : MUON_ERR_CUDA; }

int get_ctx(DeviceCtx** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MUON_ERR_CUDA;
  auto it = g_ctx.find(dev);
  if (it != g_ctx.end()) {
    *out = it->second.get();
    return MUON_OK;
  }
  cudaDeviceProp prop;
  if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return MUON_ERR_CUDA;
  if (prop.major != 10) return MUON_ERR_UNSUPPORTED;   // built for sm_100a only
  if (!encode_fn()) return MUON_ERR_UNSUPPORTED;
  std::unique_ptr<DeviceCtx> ctx(new DeviceCtx());
  ctx->device = dev;
  ctx->num_sms = prop.multiProcessorCount;
  if (cudaMalloc(&ctx->status, sizeof(int)) != cudaSuccess) return MUON_ERR_NOMEM;
  if (cudaMemset(ctx->status, 0, sizeof(int)) != cudaSuccess) return MUON_ERR_CUDA;
  if (ns_gemm_setup(dev) != cudaSuccess) return MUON_ERR_CUDA;
  ctx->max_pairs = ns_gemm_max_pairs();
  if (ctx->max_pairs < 1) ctx->max_pairs = std::max(1, prop.multiProcessorCount / 2);
  ctx->k1_blocks_per_sm = k1_blocks_per_sm();   // persistent: as many CTAs as fit
  ctx->adamw_blocks_per_sm = adamw_blocks_per_sm();
  *out = ctx.get();
  g_ctx[dev] = std::move(ctx);
  return MUON_OK;
}

unsigned long long limit_ns() {
  if (!g_limit_from_env) {
    g_limit_from_env = true;
    const char* s = std::getenv("MUON_SPIN_LIMIT_NS");
    if (s && *s) g_limit_ns = std::strtoull(s, nullptr, 10);
  }
  return g_limit_ns;
}

// Gram / poly tiles (TILE_M x BN, one per CTA pair): only tiles holding some
// entry on or above the diagonal.
void sym_tiles(std::vector<NsTile>& t, int prob, long long m, int kc, int op) {
  for (long long i0 = 0; i0 < m; i0 += TILE_M)
    for (long long j0 = 0; j0 < m; j0 += BN)
      if (std::min(j0 + BN - 1, m - 1) >= i0) t.push_back({prob, (int)i0, (int)j0, kc, op, -1, 0, -1});
}

void full_tiles(std::vector<NsTile>& t, int prob, long long m, long long n, int kc) {
  for (long long i0 = 0; i0 < m; i0 += TILE_M)
    for (long long j0 = 0; j0 < n; j0 += BN)
      t.push_back({prob, (int)i0, (int)j0, kc, OP_UPDATE, -1, 0, -1});
}

// The chain launch of ns_steps iterations: every Gram, polynomial and update
// tile except the last update's, phase after phase (phase q = 3 k + {0 Gram,
// 1 polynomial, 2 update} of iteration k), each phase listing the matrices
// in one order, costliest first, so that the static round-robin share of
// the pairs ends evenly and each matrix's phases come in sequence.  A tile
// of phase q > 0 of matrix i waits for counter (q-1) n + i to reach 16 x the
// tiles of phase q-1 of matrix i (the 8 epilogue warps of both CTAs of a
// pair count each tile once each); every tile counts itself in q n + i.
// Problem indices address the plan's five problem arrays laid end to end:
// Gram from X[0] at 0, Gram from X[1] at n, update from X[0] at 2n, update
// from X[1] at 3n, polynomial at 4n.
std::vector<NsTile> chain_tiles(const std::vector<Geom>& geom, int ns_steps) {
  const int n = (int)geom.size();
  std::vector<int> order(n);
  for (int i = 0; i < n; ++i) order[i] = i;
  auto cost = [&](int i) { return (double)geom[i].m * geom[i].m * (3.0 * geom[i].n + geom[i].m); };
  std::stable_sort(order.begin(), order.end(), [&](int a, int b) { return cost(a) > cost(b); });
  std::vector<NsTile> out, one;
  std::vector<int> prev_count(n, 0), count(n, 0);
  const int nphases = 3 * ns_steps - 1;
  for (int q = 0; q < nphases; ++q) {
    const int kind = q % 3, par = (q / 3) & 1;
    for (int i : order) {
      const Geom& g = geom[i];
      one.clear();
      if (kind == 0) sym_tiles(one, par * n + i, g.m, (int)cdiv(g.n, BK), OP_GRAM);
      else if (kind == 1) sym_tiles(one, 4 * n + i, g.m, (int)cdiv(g.m, BK), OP_POLY);
      else full_tiles(one, (2 + par) * n + i, g.m, g.n, (int)cdiv(g.m, BK));
      for (NsTile& t : one) {
        t.wait_idx = q > 0 ? (q - 1) * n + i : -1;
        t.wait_need = q > 0 ? 2 * EPI_WARPS * prev_count[i] : 0;
        t.done_idx = q * n + i;
      }
      count[i] = (int)one.size();
      out.insert(out.end(), one.begin(), one.end());
    }
    prev_count = count;
  }
  return out;
}

// K1 work queue.  Pass-2 items of a matrix wait until its norm is known,
// i.e. until every one of its pass-1 items has finished, so they are queued
// only once `slack` further pass-1 items (of later matrices) have been
// queued: by the time the persistent CTAs reach them, the matrix's last
// pass-1 items are done.  Half the number of resident CTAs is about right;
// much more slack lets g and buf drop out of L2 before pass 2 reads them
// again.  Pass-2 runs are inserted between single pass-1 items, so they
// spread evenly through the queue.
void k1_items(std::vector<K1Item>& items, const std::vector<K1Info>& info, long long slack) {
  const int n = (int)info.size();
  std::vector<long long> end1(n);   // pass-1 items queued when matrix i's pass 1 ends
  long long queued = 0;
  int next2 = 0;                    // first matrix whose pass 2 is not queued yet
  auto p2 = [&](int i) {
    for (int t = 0; t < info[i].nitems; ++t) items.push_back({i | K1_PASS2, t});
  };
  for (int i = 0; i < n; ++i) {
    for (int t = 0; t < info[i].nitems; ++t) {
      items.push_back({i, t});
      ++queued;
      while (next2 < i && queued - end1[next2] >= slack) p2(next2++);
    }
    end1[i] = queued;
  }
  while (next2 < n) p2(next2++);
}

std::vector<K1Info> k1_infos(const std::vector<Geom>& geom, const std::vector<long long>& ldx) {
  std::vector<K1Info> info;
  int part = 0;
  for (size_t i = 0; i < geom.size(); ++i) {
    K1Info k;
    k.r = geom[i].r;
    k.c = geom[i].c;
    k.ldx = ldx[i];
    k.tiles_c = (int)cdiv(k.c, K1_TILE);
    k.ntiles = (int)(cdiv(k.r, K1_TILE) * k.tiles_c);
    k.nitems = (int)cdiv(k.ntiles, K1_GROUP);
    k.part0 = part;
    k.transposed = geom[i].transposed;
    part += k.nitems;
    info.push_back(k);
  }
  return info;
}

// Tile lists of the three GEMM phases for a shape set.
struct TileLists {
  std::vector<NsTile> gram, poly, upd;
};

TileLists plan_tiles(const std::vector<Geom>& geom) {
  TileLists t;
  const int n = (int)geom.size();
  for (int i = 0; i < n; ++i) sym_tiles(t.gram, i, geom[i].m, (int)cdiv(geom[i].n, BK), OP_GRAM);
  // Longest reduction first so the static round-robin ends evenly.
  std::stable_sort(t.gram.begin(), t.gram.end(),
                   [](const NsTile& x, const NsTile& y) { return x.kc > y.kc; });
  for (int i = 0; i < n; ++i) sym_tiles(t.poly, i, geom[i].m, (int)cdiv(geom[i].m, BK), OP_POLY);
  for (int i = 0; i < n; ++i) full_tiles(t.upd, i, geom[i].m, geom[i].n, (int)cdiv(geom[i].m, BK));
  return t;
}

// Byte offsets of every scratch region inside the plan's one allocation.
struct Layout {
  long long xel = 0, ael = 0;   // elements of all iterates / all m x m matrices
  size_t x0 = 0, x1 = 0, a = 0, b = 0, probs = 0, gt = 0, pt = 0, ut = 0;
  size_t k1info = 0, k1items = 0, counters = 0, partials = 0, norms = 0;
  size_t k1tiles = 0;
  size_t total = 0;
  std::vector<size_t> guards;
};

Layout plan_layout(const std::vector<Geom>& geom, bool with_ns, const TileLists* t) {
  Layout L;
  Arena a;
  const int n = (int)geom.size();
  for (const Geom& g : geom) {
    L.xel += round_up(g.m * g.ldx, 128);
    L.ael += round_up(g.m * g.lda, 128);
    L.k1tiles += cdiv(g.r, K1_TILE) * cdiv(g.c, K1_TILE);
  }
  L.x0 = a.take(L.xel * 2);
  if (with_ns) {
    L.x1 = a.take(L.xel * 2);
    L.a = a.take(L.ael * 2);
    L.b = a.take(L.ael * 2);
    L.probs = a.take(sizeof(NsProblem) * n * 5, 128);
    L.gt = a.take(sizeof(NsTile) * t->gram.size());
    L.pt = a.take(sizeof(NsTile) * t->poly.size());
    L.ut = a.take(sizeof(NsTile) * t->upd.size());
  }
  L.k1info = a.take(sizeof(K1Info) * n);
  L.k1items = a.take(sizeof(K1Item) * 2 * L.k1tiles);
  // K1 counters, then one chain counter per (phase, matrix)
  L.counters = a.take(sizeof(int) * (1 + 2 * n + 3 * (size_t)kMaxSteps * n));
  L.partials = a.take(sizeof(double) * L.k1tiles);
  L.norms = a.take(sizeof(double) * n);
  L.total = a.off;
  L.guards = a.guards;
  return L;
}

size_t plan_bytes(const std::vector<Geom>& geom, bool with_ns) {
  TileLists t;
  if (with_ns) t = plan_tiles(geom);
  return plan_layout(geom, with_ns, &t).total;
}

std::vector<Geom> make_geom(const int64_t* shapes, int n) {
  std::vector<Geom> geom(n);
  for (int i = 0; i < n; ++i) {
    Geom& g = geom[i];
    g.r = shapes[2 * i];
    g.c = shapes[2 * i + 1];
    g.transposed = g.r > g.c;
    g.m = std::min(g.r, g.c);
    g.n = std::max(g.r, g.c);
    g.ldx = round_up(g.n, 8);
    g.lda = round_up(g.m, 8);
  }
  return geom;
}

int upload_phase(NsPhase& ph, char* base, size_t prob_off, size_t tile_off,
                 const std::vector<NsProblem>& probs, const std::vector<NsTile>& tiles) {
  ph.probs = reinterpret_cast<NsProblem*>(base + prob_off);
  ph.tiles = reinterpret_cast<NsTile*>(base + tile_off);
  ph.ntiles = (int)tiles.size();
  if (cudaMemcpy(ph.probs, probs.data(), sizeof(NsProblem) * probs.size(), cudaMemcpyHostToDevice) !=
      cudaSuccess)
    return MUON_ERR_CUDA;
  if (!tiles.empty() &&
      cudaMemcpy(ph.tiles, tiles.data(), sizeof(NsTile) * tiles.size(), cudaMemcpyHostToDevice) !=
          cudaSuccess)
    return MUON_ERR_CUDA;
  return MUON_OK;
}

// Builds the scratch memory, tensor maps, tile lists and work queue for a
// shape set.  with_ns=false builds only the first-kernel part.
int build_plan(const std::vector<Geom>& geom, bool with_ns, long long k1_slack,
               std::unique_ptr<Plan>* out) {
  std::unique_ptr<Plan> P(new Plan());
  P->geom = geom;
  const int n = (int)geom.size();
  TileLists tl;
  if (with_ns) tl = plan_tiles(geom);
  const Layout lay = plan_layout(geom, with_ns, &tl);
  if (cudaMalloc(&P->mem.ptr, lay.total) != cudaSuccess) {
    cudaGetLastError();
    return MUON_ERR_NOMEM;
  }
  P->mem.bytes = lay.total;
  char* base = P->mem.ptr;
  P->guards = lay.guards;
  for (size_t g : lay.guards)
    if (cudaMemset(base + g, kGuardByte, kGuardBytes) != cudaSuccess) return MUON_ERR_CUDA;
  long long xel = 0, ael = 0;
  P->x_off.resize(n);
  P->a_off.resize(n);
  for (int i = 0; i < n; ++i) {
    P->x_off[i] = xel;
    P->a_off[i] = ael;
    xel += round_up(geom[i].m * geom[i].ldx, 128);
    ael += round_up(geom[i].m * geom[i].lda, 128);
  }
  P->X[0] = reinterpret_cast<__nv_bfloat16*>(base + lay.x0);
  if (with_ns) {
    P->X[1] = reinterpret_cast<__nv_bfloat16*>(base + lay.x1);
    P->A = reinterpret_cast<__nv_bfloat16*>(base + lay.a);
    P->B = reinterpret_cast<__nv_bfloat16*>(base + lay.b);
    const size_t prob_off = lay.probs;
    const std::vector<NsTile>& gt = tl.gram;
    const std::vector<NsTile>& pt = tl.poly;
    const std::vector<NsTile>& ut = tl.upd;
    const size_t gt_off = lay.gt, pt_off = lay.pt, ut_off = lay.ut;

    std::vector<NsProblem> pr(n);
    for (int par = 0; par < 2; ++par) {
      // Gram: A = X X^T from X[par]
      for (int i = 0; i < n; ++i) {
        const Geom& g = geom[i];
        NsProblem& q = pr[i];
        std::memset(&q, 0, sizeof(q));
        const __nv_bfloat16* x = P->X[par] + P->x_off[i];
        if (!make_map(&q.tmA, x, g.m, g.n, g.ldx)) return MUON_ERR_CUDA;
        q.tmB = q.tmA;
        q.out = P->A + P->a_off[i];
        q.ld_out = g.lda;
        if (!make_out_map(&q.tmOut, q.out, g.m, g.m, g.lda)) return MUON_ERR_CUDA;
        q.M = (int)g.m;
        q.N = (int)g.m;
        q.K = (int)g.n;
        q.slot = i;
      }
      int rc = upload_phase(P->gram[par], base, prob_off + sizeof(NsProblem) * n * par, gt_off, pr, gt);
      if (rc) return rc;
      // Update: X[1-par] = a X[par] + B X[par]
      for (int i = 0; i < n; ++i) {
        const Geom& g = geom[i];
        NsProblem& q = pr[i];
        std::memset(&q, 0, sizeof(q));
        const __nv_bfloat16* x = P->X[par] + P->x_off[i];
        if (!make_map(&q.tmA, P->B + P->a_off[i], g.m, g.m, g.lda)) return MUON_ERR_CUDA;
        if (!make_map(&q.tmB, x, g.m, g.n, g.ldx)) return MUON_ERR_CUDA;
        q.epi = x;
        q.ld_epi = g.ldx;
        q.out = P->X[1 - par] + P->x_off[i];
        q.ld_out = g.ldx;
        if (!make_out_map(&q.tmOut, q.out, g.m, g.n, g.ldx, true)) return MUON_ERR_CUDA;
        q.M = (int)g.m;
        q.N = (int)g.n;
        q.K = (int)g.m;
        q.transposed = g.transposed;
        q.ld_final = g.c;
        q.slot = i;
      }
      rc = upload_phase(P->upd[par], base, prob_off + sizeof(NsProblem) * n * (2 + par), ut_off, pr, ut);
      if (rc) return rc;
    }
    // Poly: B = b A + c A A^T
    for (int i = 0; i < n; ++i) {
      const Geom& g = geom[i];
      NsProblem& q = pr[i];
      std::memset(&q, 0, sizeof(q));
      const __nv_bfloat16* am = P->A + P->a_off[i];
      if (!make_map(&q.tmA, am, g.m, g.m, g.lda)) return MUON_ERR_CUDA;
      q.tmB = q.tmA;
      q.epi = am;
      q.ld_epi = g.lda;
      q.out = P->B + P->a_off[i];
      q.ld_out = g.lda;
      if (!make_out_map(&q.tmOut, q.out, g.m, g.m, g.lda)) return MUON_ERR_CUDA;
      q.M = (int)g.m;
      q.N = (int)g.m;
      q.K = (int)g.m;
      q.slot = i;
    }
    int rc = upload_phase(P->poly, base, prob_off + sizeof(NsProblem) * n * 4, pt_off, pr, pt);
    if (rc) return rc;
  }
  // First kernel.
  std::vector<long long> ldx(n);
  for (int i = 0; i < n; ++i) ldx[i] = geom[i].ldx;
  std::vector<K1Info> info = k1_infos(geom, ldx);
  std::vector<K1Item> items;
  k1_items(items, info, k1_slack);
  P->k1.n = n;
  P->k1.info = reinterpret_cast<K1Info*>(base + lay.k1info);
  P->k1.items = reinterpret_cast<K1Item*>(base + lay.k1items);
  P->k1.nitems = (int)items.size();
  P->k1.counters = reinterpret_cast<int*>(base + lay.counters);
  P->k1.partials = reinterpret_cast<double*>(base + lay.partials);
  P->k1.norms = reinterpret_cast<double*>(base + lay.norms);
  P->k1.npartials = (int)lay.k1tiles;
  P->deps = P->k1.counters + 1 + 2 * n;
  if (cudaMemcpy(P->k1.info, info.data(), sizeof(K1Info) * n, cudaMemcpyHostToDevice) != cudaSuccess)
    return MUON_ERR_CUDA;
  if (cudaMemcpy(P->k1.items, items.data(), sizeof(K1Item) * items.size(), cudaMemcpyHostToDevice) !=
      cudaSuccess)
    return MUON_ERR_CUDA;
  *out = std::move(P);
  return MUON_OK;
}

int check_shapes(const int64_t* shapes, int n) {
  if (n < 0 || n > (1 << 20)) return MUON_ERR_INVALID_ARG;
  if (n > 0 && !shapes) return MUON_ERR_INVALID_ARG;
  for (int i = 0; i < n; ++i) {
    const long long r = shapes[2 * i], c = shapes[2 * i + 1];
    if (r <= 0 || c <= 0) return MUON_ERR_INVALID_ARG;
    if (r * c >= (1ll << 31) || r >= (1ll << 30) || c >= (1ll << 30)) return MUON_ERR_UNSUPPORTED;
  }
  return MUON_OK;
}

int check_coeffs(const float* coeffs, float* co) {
  const float* src = coeffs ? coeffs : kDefaultCoeffs;
  for (int i = 0; i < 3; ++i) {
    if (!std::isfinite(src[i])) return MUON_ERR_INVALID_ARG;
    co[i] = src[i];
  }
  return MUON_OK;
}

// Pass-1 items queued between a matrix's pass 1 and its pass 2: half the
// first kernel's resident CTAs.
long long k1_queue_slack(const DeviceCtx* ctx) {
  return std::max(1, ctx->num_sms * ctx->k1_blocks_per_sm / 2);
}

int get_plan(DeviceCtx* ctx, std::vector<long long> key, const std::vector<Geom>& geom, bool with_ns,
             Plan** out) {
  auto it = ctx->plans.find(key);
  if (it != ctx->plans.end()) {
    *out = it->second.get();
    return MUON_OK;
  }
  std::unique_ptr<Plan> P;
  int rc = build_plan(geom, with_ns, k1_queue_slack(ctx), &P);
  if (rc) return rc;
  *out = P.get();
  ctx->plans[key] = std::move(P);
  return MUON_OK;
}

// Persistent GEMM grid: two CTAs (one cluster) per tile, at most one per SM.
int pair_grid(DeviceCtx* ctx, int ntiles) { return 2 * std::max(1, std::min(ntiles, ctx->max_pairs)); }

int k1_grid(DeviceCtx* ctx, int nitems) {
  return std::max(1, std::min(nitems, ctx->num_sms * ctx->k1_blocks_per_sm));
}

// zero_deps: how many chain counters after the K1 counters to zero as well
// (the same memset), for the chain launch that follows.
int run_k1(DeviceCtx* ctx, Plan* P, const K1Ptrs* ptrs, int mode, float beta, int nesterov,
           cudaStream_t stream, int zero_deps = 0) {
  const int n = P->k1.n;
  if (cudaMemsetAsync(P->k1.counters, 0, sizeof(int) * (1 + 2 * n + (size_t)zero_deps), stream) !=
      cudaSuccess)
    return MUON_ERR_CUDA;
  static thread_local K1Launch L;   // large (12 KB); kept off the stack
  L.info = P->k1.info;
  L.items = P->k1.items;
  L.nitems = P->k1.nitems;
  L.n = n;
  L.npartials = P->k1.npartials;
  L.mode = mode;
  L.nesterov = nesterov;
  L.beta = beta;
  L.counter = P->k1.counters;
  L.done = P->k1.counters + 1;
  L.ready = P->k1.counters + 1 + n;
  L.partials = P->k1.partials;
  L.norms = P->k1.norms;
  L.limit_ns = limit_ns();
  L.status = ctx->status;
  for (int i = 0; i < n; ++i) L.ptrs[i] = ptrs[i];
  ProfScope ps(PK_K1, stream);
  return cuda_err(launch_k1(L, k1_grid(ctx, L.nitems), stream));
}

// The chain tile list of ns_steps iterations for this plan (built and
// uploaded on first use; blocking copies, so before any capture).
int get_chain(Plan* P, int ns_steps, const Plan::Chain** out) {
  auto it = P->chains.find(ns_steps);
  if (it == P->chains.end()) {
    std::vector<NsTile> tiles = chain_tiles(P->geom, ns_steps);
    Plan::Chain c;
    c.ntiles = (int)tiles.size();
    c.mem.reset(new DevBlock());
    const size_t bytes = sizeof(NsTile) * std::max<size_t>(1, tiles.size());
    if (cudaMalloc(&c.mem->ptr, bytes) != cudaSuccess) {
      cudaGetLastError();
      return MUON_ERR_NOMEM;
    }
    c.mem->bytes = bytes;
    if (!tiles.empty() &&
        cudaMemcpy(c.mem->ptr, tiles.data(), sizeof(NsTile) * tiles.size(), cudaMemcpyHostToDevice) !=
            cudaSuccess)
      return MUON_ERR_CUDA;
    it = P->chains.emplace(ns_steps, std::move(c)).first;
  }
  *out = &it->second;
  return MUON_OK;
}

// Which launch sequence runs the iterations.  The chain launch saves each
// phase's launch and lets a matrix's next phase start as soon as its own
// tiles are done, but its kernel carries all three epilogues; a per-phase
// launch runs a kernel specialised to one operation, 5-9% faster per tile
// (measured on GPT-2 124M).  The chain wins where the phases are short: when
// the largest phase (the X update) has at most two waves of tiles for the
// resident CTA pairs (GPT-2 block: 0.266 vs 0.300 ms of Newton-Schulz; one
// 256 x 256 matrix: 0.114 vs 0.180 ms; GPT-2 124M, 17.5 waves: 1.125 vs
// 1.074 ms).
bool use_chain(const DeviceCtx* ctx, const Plan* P, int ns_steps) {
  return ns_steps > 0 && P->upd[0].ntiles <= 2 * ctx->max_pairs;
}

// Chain counters run_k1 must zero before the chain launch of ns_steps.
int chain_deps(const DeviceCtx* ctx, const Plan* P, int ns_steps) {
  return use_chain(ctx, P, ns_steps) ? (3 * ns_steps - 1) * (int)P->geom.size() : 0;
}

// The Newton-Schulz iterations, then the last update, which writes
// `final_mode` through F (through the parameter tensor maps `pmaps` when
// given).  Either one chain launch for every phase but the last update (its
// counters zeroed by run_k1 with zero_deps = chain_deps), or one launch per
// phase (use_chain).
int run_ns(DeviceCtx* ctx, Plan* P, int ns_steps, const float* co, int final_mode,
           const FinalTable* F, cudaStream_t stream, const CUtensorMap* pmaps = nullptr,
           float* const* mirrors = nullptr, int n_mirrors = 0) {
  const int n = (int)P->geom.size();
  NsLaunch L;
  L.deps = nullptr;
  L.ndeps = 0;
  L.nprobs = n;
  L.pmaps = nullptr;
  L.mirrors = nullptr;
  L.n_mirrors = 0;
  L.mirror_stride = n;
  L.ca = co[0];
  L.cb = co[1];
  L.cc = co[2];
  L.limit_ns = limit_ns();
  L.status = ctx->status;
  L.final_mode = FINAL_NONE;
  cudaError_t e = cudaSuccess;
  auto phase = [&](const NsPhase& ph, int op, int kind) {
    L.probs = ph.probs;
    L.tiles = ph.tiles;
    L.ntiles = ph.ntiles;
    ProfScope ps(kind, stream);
    e = launch_ns_gemm(L, nullptr, pair_grid(ctx, L.ntiles), stream, op);
  };
  bool chained = false;
  if (use_chain(ctx, P, ns_steps)) {
    const Plan::Chain* chain = nullptr;
    int rc = get_chain(P, ns_steps, &chain);
    if (rc) return rc;
    L.probs = P->gram[0].probs;            // the five problem arrays, end to end
    L.nprobs = 5 * n;
    L.deps = P->deps;
    L.ndeps = 3 * kMaxSteps * n;
    L.tiles = reinterpret_cast<const NsTile*>(chain->mem->ptr);
    L.ntiles = chain->ntiles;
    {
      ProfScope ps(PK_CHAIN, stream);
      e = launch_ns_gemm(L, nullptr, pair_grid(ctx, L.ntiles), stream, /*op=*/-1);
    }
    L.nprobs = n;
    L.deps = nullptr;
    L.ndeps = 0;
    if (e == cudaErrorCooperativeLaunchTooLarge) {
      // The device cannot hold every CTA pair at once right now (it is shared
      // with another context): nothing was launched, so run the phases as
      // separate launches instead.
      cudaGetLastError();
      e = cudaSuccess;
    } else if (e != cudaSuccess) {
      return MUON_ERR_CUDA;
    } else {
      chained = true;
    }
  }
  if (!chained) {
    for (int s = 0; s < ns_steps; ++s) {
      const int par = s & 1;
      phase(P->gram[par], OP_GRAM, PK_GRAM);
      if (e != cudaSuccess) return MUON_ERR_CUDA;
      phase(P->poly, OP_POLY, PK_POLY);
      if (e != cudaSuccess) return MUON_ERR_CUDA;
      if (s == ns_steps - 1) break;
      phase(P->upd[par], OP_UPDATE, PK_UPDATE);
      if (e != cudaSuccess) return MUON_ERR_CUDA;
    }
  }
  const NsPhase& last = P->upd[(ns_steps - 1) & 1];
  L.probs = last.probs;
  L.tiles = last.tiles;
  L.ntiles = last.ntiles;
  L.final_mode = final_mode;
  L.pmaps = pmaps;
  L.mirrors = mirrors;
  L.n_mirrors = n_mirrors;
  {
    ProfScope ps(PK_FINAL, stream);
    e = launch_ns_gemm(L, F, pair_grid(ctx, L.ntiles), stream, OP_UPDATE);
  }
  return e == cudaSuccess ? MUON_OK : MUON_ERR_CUDA;
}

int run_apply(Plan* P, int mode, void* const* dst, const float* scale, cudaStream_t stream) {
  static thread_local ApplyLaunch A;
  A.info = P->k1.info;
  A.n = P->k1.n;
  A.mode = mode;
  for (int i = 0; i < A.n; ++i) {
    A.ptrs[i].g = nullptr;
    A.ptrs[i].buf = nullptr;
    A.ptrs[i].x0 = P->X[0] + P->x_off[i];
    A.dst[i] = dst[i];
    A.scale[i] = scale ? scale[i] : 0.f;
  }
  ProfScope ps(PK_APPLY, stream);
  return cuda_err(launch_apply(A, stream));
}

std::vector<long long> shape_key(char kind, const std::vector<Geom>& geom) {
  std::vector<long long> key;
  key.push_back(kind);
  for (const Geom& g : geom) {
    key.push_back(g.r);
    key.push_back(g.c);
  }
  return key;
}

// Tensor maps over the caller's parameters for the TMA path of the last X
// update.  They depend on the pointers, so each plan keeps the maps of the
// last kParamMapSets pointer sets, each in its own device block that is
// written once, before any kernel reads it, and never changed while cached:
// a call with a cached pointer set (a training loop alternating a few models
// or parameter copies of one shape set) reuses its block and does not
// synchronise.  Only when a new set evicts the least recently used block is
// the stream synchronised first, since kernels queued earlier may still read
// that block.  Shapes whose row pitch is not a multiple of 16 bytes use the
// register path (*out = nullptr).
constexpr size_t kParamMapSets = 8;

int ensure_param_maps(Plan* P, float* const* params, int n, cudaStream_t stream,
                      const CUtensorMap** out) {
  *out = nullptr;
  for (int i = 0; i < n; ++i)
    if (P->geom[i].c % 4 != 0) return MUON_OK;
  std::vector<const void*> want(params, params + n);
  for (size_t k = 0; k < P->pmaps.size(); ++k) {
    if (P->pmaps[k].ptrs != want) continue;
    if (k != 0) std::rotate(P->pmaps.begin(), P->pmaps.begin() + k, P->pmaps.begin() + k + 1);
    *out = reinterpret_cast<const CUtensorMap*>(P->pmaps[0].mem->ptr);
    return MUON_OK;
  }
  std::vector<CUtensorMap> maps(n);
  for (int i = 0; i < n; ++i)
    if (!make_param_map(&maps[i], params[i], P->geom[i].r, P->geom[i].c)) return MUON_ERR_CUDA;
  std::unique_ptr<DevBlock> blk;
  if (P->pmaps.size() >= kParamMapSets) {
    // The least recently used block may still be read by queued kernels.
    if (cudaStreamSynchronize(stream) != cudaSuccess) return MUON_ERR_CUDA;
    blk = std::move(P->pmaps.back().mem);
    P->pmaps.pop_back();
  } else {
    blk.reset(new DevBlock());
    if (cudaMalloc(&blk->ptr, sizeof(CUtensorMap) * n) != cudaSuccess) {
      cudaGetLastError();
      return MUON_ERR_NOMEM;
    }
    blk->bytes = sizeof(CUtensorMap) * n;
  }
  if (cudaMemcpy(blk->ptr, maps.data(), sizeof(CUtensorMap) * n, cudaMemcpyHostToDevice) !=
      cudaSuccess)
    return MUON_ERR_CUDA;
  P->pmaps.insert(P->pmaps.begin(), Plan::ParamMaps{want, std::move(blk)});
  *out = reinterpret_cast<const CUtensorMap*>(P->pmaps[0].mem->ptr);
  return MUON_OK;
}

// Uploads the group's mirror table (n_mirrors x n device pointers, row k
// contiguous) unless the plan already holds the same one.
int ensure_mirror_table(Plan* P, float* const* tab, int count, cudaStream_t stream,
                        float* const** out) {
  *out = nullptr;
  if (count == 0) return MUON_OK;
  std::vector<const void*> want(tab, tab + count);
  if (P->mirror_mem.ptr && P->mirror_for == want) {
    *out = reinterpret_cast<float* const*>(P->mirror_mem.ptr);
    return MUON_OK;
  }
  // An earlier launch may still read the old table.
  if (P->mirror_mem.ptr && cudaStreamSynchronize(stream) != cudaSuccess) return MUON_ERR_CUDA;
  const size_t bytes = sizeof(float*) * (size_t)count;
  if (P->mirror_mem.bytes < bytes) {
    if (P->mirror_mem.ptr) {
      cudaFree(P->mirror_mem.ptr);
      P->mirror_mem.ptr = nullptr;
      P->mirror_mem.bytes = 0;
    }
    if (cudaMalloc(&P->mirror_mem.ptr, bytes) != cudaSuccess) {
      cudaGetLastError();
      return MUON_ERR_NOMEM;
    }
    P->mirror_mem.bytes = bytes;
  }
  if (cudaMemcpy(P->mirror_mem.ptr, tab, bytes, cudaMemcpyHostToDevice) != cudaSuccess)
    return MUON_ERR_CUDA;
  P->mirror_for = want;
  *out = reinterpret_cast<float* const*>(P->mirror_mem.ptr);
  return MUON_OK;
}

int step_group(DeviceCtx* ctx, float* const* params, const float* const* grads, float* const* bufs,
               const int64_t* shapes, int n, float lr, float beta, int nesterov, int ns_steps,
               const float* co, cudaStream_t stream, float* const* mirror_tab = nullptr,
               int n_mirrors = 0) {
  std::vector<Geom> geom = make_geom(shapes, n);
  Plan* P = nullptr;
  int rc = get_plan(ctx, shape_key('S', geom), geom, true, &P);
  if (rc) return rc;
  std::vector<K1Ptrs> ptrs(n);
  static thread_local FinalTable F;
  for (int i = 0; i < n; ++i) {
    ptrs[i].g = grads[i];
    ptrs[i].buf = bufs[i];
    ptrs[i].x0 = P->X[0] + P->x_off[i];
    F.ptr[i] = params[i];
    const double s = std::sqrt(std::max(1.0, (double)geom[i].r / (double)geom[i].c));
    F.scale[i] = (float)((double)lr * s);
  }
  rc = run_k1(ctx, P, ptrs.data(), K1_MOMENTUM, beta, nesterov, stream,
              chain_deps(ctx, P, ns_steps));
  if (rc) return rc;
  if (ns_steps == 0) {
    std::vector<void*> dst(params, params + n);
    return run_apply(P, FINAL_PARAM, dst.data(), F.scale, stream);
  }
  const CUtensorMap* pmaps = nullptr;
  rc = ensure_param_maps(P, params, n, stream, &pmaps);
  if (rc) return rc;
  float* const* mirrors = nullptr;
  if (n_mirrors > 0) {
    if (pmaps == nullptr) return MUON_ERR_UNSUPPORTED;   // checked by the caller already
    rc = ensure_mirror_table(P, mirror_tab, n_mirrors * n, stream, &mirrors);
    if (rc) return rc;
  }
  return run_ns(ctx, P, ns_steps, co, FINAL_PARAM, &F, stream, pmaps, mirrors, n_mirrors);
}

}  // namespace

unsigned long long current_wait_limit_ns() {
  std::lock_guard<std::mutex> lock(g_mutex);
  return limit_ns();
}

}  // namespace muon

using namespace muon;

extern "C" {

int muon_step_mirrored(float* const* params, const float* const* grads, float* const* bufs,
                       const int64_t* shapes, int n, float lr, float beta, int nesterov,
                       int ns_steps, const float* coeffs, float* const* mirrors, int n_mirrors,
                       void* stream) {
  int rc = check_shapes(shapes, n);
  if (rc) return rc;
  if (n_mirrors < 0 || n_mirrors > MUON_MAX_MIRRORS) return MUON_ERR_INVALID_ARG;
  if (n == 0) return MUON_OK;
  if (!params || !grads || !bufs) return MUON_ERR_INVALID_ARG;
  if (!std::isfinite(lr) || !std::isfinite(beta)) return MUON_ERR_INVALID_ARG;
  if (ns_steps < 0 || ns_steps > kMaxSteps) return MUON_ERR_INVALID_ARG;
  float co[3];
  rc = check_coeffs(coeffs, co);
  if (rc) return rc;
  for (int i = 0; i < n; ++i) {
    if (!params[i] || !grads[i] || !bufs[i]) return MUON_ERR_INVALID_ARG;
    if (!aligned16(params[i]) || !aligned16(grads[i]) || !aligned16(bufs[i]))
      return MUON_ERR_UNSUPPORTED;
  }
  if (n_mirrors > 0) {
    if (!mirrors) return MUON_ERR_INVALID_ARG;
    for (long long j = 0; j < (long long)n_mirrors * n; ++j) {
      if (!mirrors[j]) return MUON_ERR_INVALID_ARG;
      if (!aligned16(mirrors[j])) return MUON_ERR_UNSUPPORTED;
    }
    // Mirrors are written from the shared-memory parameter blocks of the
    // last X update, which need at least one iteration and c % 4 == 0.
    if (ns_steps < 1) return MUON_ERR_UNSUPPORTED;
    for (int i = 0; i < n; ++i)
      if (shapes[2 * i + 1] % 4 != 0) return MUON_ERR_UNSUPPORTED;
  }
  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceCtx* ctx = nullptr;
  rc = get_ctx(&ctx);
  if (rc) return rc;
  std::vector<float*> tab;
  for (int g0 = 0; g0 < n; g0 += MUON_MAX_GROUP) {
    const int gn = std::min(MUON_MAX_GROUP, n - g0);
    tab.assign((size_t)n_mirrors * gn, nullptr);
    for (int k = 0; k < n_mirrors; ++k)
      for (int i = 0; i < gn; ++i) tab[(size_t)k * gn + i] = mirrors[(size_t)k * n + g0 + i];
    rc = step_group(ctx, params + g0, grads + g0, bufs + g0, shapes + 2 * g0, gn, lr, beta, nesterov,
                    ns_steps, co, static_cast<cudaStream_t>(stream), tab.data(), n_mirrors);
    if (rc) return rc;
  }
  return MUON_OK;
}

int muon_step(float* const* params, const float* const* grads, float* const* bufs,
              const int64_t* shapes, int n, float lr, float beta, int nesterov, int ns_steps,
              const float* coeffs, void* stream) {
  return muon_step_mirrored(params, grads, bufs, shapes, n, lr, beta, nesterov, ns_steps, coeffs,
                            nullptr, 0, stream);
}

int muon_adamw_step(float* const* params, const float* const* grads, float* const* exp_avgs,
                    float* const* exp_avg_sqs, const int64_t* numels, const unsigned char* decay,
                    int n, int64_t step, double lr, double beta1, double beta2, double eps,
                    double weight_decay, void* stream) {
  if (n < 0) return MUON_ERR_INVALID_ARG;
  if (n == 0) return MUON_OK;
  if (!params || !grads || !exp_avgs || !exp_avg_sqs || !numels) return MUON_ERR_INVALID_ARG;
  if (step < 1) return MUON_ERR_INVALID_ARG;
  for (double h : {lr, beta1, beta2, eps, weight_decay})
    if (!std::isfinite(h)) return MUON_ERR_INVALID_ARG;
  if (lr < 0 || eps < 0 || weight_decay < 0 || beta1 < 0 || beta1 >= 1 || beta2 < 0 || beta2 >= 1)
    return MUON_ERR_INVALID_ARG;
  constexpr long long kMaxNumel = (1ll << 40);
  int nonempty = 0;
  for (int i = 0; i < n; ++i) {
    if (numels[i] < 0 || numels[i] > kMaxNumel) return MUON_ERR_INVALID_ARG;
    if (numels[i] == 0) continue;
    ++nonempty;
    if (!params[i] || !grads[i] || !exp_avgs[i] || !exp_avg_sqs[i]) return MUON_ERR_INVALID_ARG;
    for (const void* q : {(const void*)params[i], (const void*)grads[i], (const void*)exp_avgs[i],
                          (const void*)exp_avg_sqs[i]})
      if (reinterpret_cast<uintptr_t>(q) & 3u) return MUON_ERR_UNSUPPORTED;   // not a float address
  }
  if (nonempty == 0) return MUON_OK;
  // Host-side constants in double, each rounded once to fp32.
  const double bc1 = 1.0 - std::pow(beta1, (double)step);
  const double bc2 = 1.0 - std::pow(beta2, (double)step);
  static thread_local AdamWLaunch L;
  L.beta1 = (float)beta1;
  L.one_minus_beta1 = (float)(1.0 - beta1);
  L.beta2 = (float)beta2;
  L.one_minus_beta2 = (float)(1.0 - beta2);
  L.step_size = (float)(lr / bc1);
  L.inv_sqrt_bc2 = (float)(1.0 / std::sqrt(bc2));
  L.eps = (float)eps;

  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceCtx* ctx = nullptr;
  int rc = get_ctx(&ctx);
  if (rc) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int max_grid = ctx->num_sms * ctx->adamw_blocks_per_sm;
  auto flush = [&]() -> int {
    if (L.n == 0) return MUON_OK;
    const int grid = std::max(1, std::min(L.nchunks, max_grid));
    ProfScope ps(PK_ADAMW, s);
    const int r = cuda_err(launch_adamw(L, grid, s));
    L.n = 0;
    L.nchunks = 0;
    return r;
  };
  L.n = 0;
  L.nchunks = 0;
  constexpr long long kMaxChunks = (1ll << 30);
  for (int i = 0; i < n; ++i) {
    if (numels[i] == 0) continue;
    const long long chunks = cdiv(numels[i], ADAMW_CHUNK);
    if (L.n == ADAMW_MAX_TENSORS || L.nchunks + chunks > kMaxChunks) {
      rc = flush();
      if (rc) return rc;
    }
    AdamWTensor& T = L.t[L.n++];
    T.p = params[i];
    T.g = grads[i];
    T.m = exp_avgs[i];
    T.v = exp_avg_sqs[i];
    T.numel = numels[i];
    T.chunk0 = L.nchunks;
    T.vec = aligned16(params[i]) && aligned16(grads[i]) && aligned16(exp_avgs[i]) &&
            aligned16(exp_avg_sqs[i]);
    T.decay = (float)(1.0 - lr * ((decay == nullptr || decay[i]) ? weight_decay : 0.0));
    T.pad_ = 0;
    L.nchunks += (int)chunks;
  }
  return flush();
}

int muon_orthogonalize(const float* x, void* out, int out_is_bf16, int64_t rows, int64_t cols,
                       int ns_steps, const float* coeffs, void* stream) {
  const int64_t shp[2] = {rows, cols};
  int rc = check_shapes(shp, 1);
  if (rc) return rc;
  if (!x || !out) return MUON_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(out)) return MUON_ERR_UNSUPPORTED;
  if (ns_steps < 0 || ns_steps > kMaxSteps) return MUON_ERR_INVALID_ARG;
  float co[3];
  rc = check_coeffs(coeffs, co);
  if (rc) return rc;
  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceCtx* ctx = nullptr;
  rc = get_ctx(&ctx);
  if (rc) return rc;
  std::vector<Geom> geom = make_geom(shp, 1);
  Plan* P = nullptr;
  rc = get_plan(ctx, shape_key('O', geom), geom, true, &P);
  if (rc) return rc;
  K1Ptrs p;
  p.g = x;
  p.buf = nullptr;
  p.x0 = P->X[0];
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  rc = run_k1(ctx, P, &p, K1_PLAIN, 0.f, 0, s, chain_deps(ctx, P, ns_steps));
  if (rc) return rc;
  const int mode = out_is_bf16 ? FINAL_OUT_BF16 : FINAL_OUT_F32;
  if (ns_steps == 0) {
    void* dst[1] = {out};
    return run_apply(P, mode, dst, nullptr, s);
  }
  static thread_local FinalTable F;
  F.ptr[0] = out;
  F.scale[0] = 0.f;
  return run_ns(ctx, P, ns_steps, co, mode, &F, s);
}

int muon_momentum_normalize(const float* const* grads, float* const* bufs, uint16_t* const* x0,
                            const int64_t* x0_ld, const int64_t* shapes, int n, float beta,
                            int nesterov, void* stream) {
  int rc = check_shapes(shapes, n);
  if (rc) return rc;
  if (n == 0) return MUON_OK;
  if (n > MUON_MAX_GROUP) return MUON_ERR_INVALID_ARG;
  if (!grads || !bufs || !x0 || !x0_ld || !std::isfinite(beta)) return MUON_ERR_INVALID_ARG;
  for (int i = 0; i < n; ++i) {
    if (!grads[i] || !bufs[i] || !x0[i]) return MUON_ERR_INVALID_ARG;
    if (!aligned16(grads[i]) || !aligned16(bufs[i]) || !aligned16(x0[i])) return MUON_ERR_UNSUPPORTED;
    const long long ncols = std::max(shapes[2 * i], shapes[2 * i + 1]);
    if (x0_ld[i] < ncols || (x0_ld[i] & 7)) return MUON_ERR_INVALID_ARG;
  }
  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceCtx* ctx = nullptr;
  rc = get_ctx(&ctx);
  if (rc) return rc;
  std::vector<Geom> geom = make_geom(shapes, n);
  std::vector<long long> key = shape_key('K', geom);
  for (int i = 0; i < n; ++i) {
    geom[i].ldx = x0_ld[i];
    key.push_back(x0_ld[i]);
  }
  Plan* P = nullptr;
  rc = get_plan(ctx, key, geom, false, &P);
  if (rc) return rc;
  std::vector<K1Ptrs> ptrs(n);
  for (int i = 0; i < n; ++i) {
    ptrs[i].g = grads[i];
    ptrs[i].buf = bufs[i];
    ptrs[i].x0 = reinterpret_cast<__nv_bfloat16*>(x0[i]);
  }
  return run_k1(ctx, P, ptrs.data(), K1_MOMENTUM, beta, nesterov, static_cast<cudaStream_t>(stream));
}

// One GEMM phase on caller buffers (stage entry points).
static int run_stage(int op, const uint16_t* opA, long long ldA, const uint16_t* opB, long long ldB,
                     long long rowsB, long long colsB, const uint16_t* epi, long long ld_epi,
                     uint16_t* out, long long ld_out, long long M, long long N, long long K, float ca,
                     float cb, float cc, void* stream) {
  DeviceCtx* ctx = nullptr;
  int rc = get_ctx(&ctx);
  if (rc) return rc;
  std::vector<long long> key = {'G', op, (long long)(uintptr_t)opA, ldA, (long long)(uintptr_t)opB, ldB,
                                rowsB, colsB, (long long)(uintptr_t)epi, ld_epi,
                                (long long)(uintptr_t)out, ld_out, M, N, K};
  Plan* P = nullptr;
  if (ctx->stage_plans.size() >= 64 && !ctx->stage_plans.count(key)) {
    // Bounded cache: older stage plans may still be read by queued kernels.
    if (cudaDeviceSynchronize() != cudaSuccess) return MUON_ERR_CUDA;
    ctx->stage_plans.clear();
  }
  auto it = ctx->stage_plans.find(key);
  if (it != ctx->stage_plans.end()) {
    P = it->second.get();
  } else {
    std::unique_ptr<Plan> np(new Plan());
    std::vector<NsTile> tiles;
    const int kc = (int)cdiv(K, BK);
    if (op == OP_UPDATE)
      full_tiles(tiles, 0, M, N, kc);
    else
      sym_tiles(tiles, 0, M, kc, op);
    const size_t bytes = 256 + sizeof(NsProblem) + sizeof(NsTile) * tiles.size();
    if (cudaMalloc(&np->mem.ptr, bytes) != cudaSuccess) {
      cudaGetLastError();
      return MUON_ERR_NOMEM;
    }
    np->mem.bytes = bytes;
    NsProblem q;
    std::memset(&q, 0, sizeof(q));
    if (!make_map(&q.tmA, opA, M, K, ldA)) return MUON_ERR_CUDA;
    if (!make_map(&q.tmB, opB, rowsB, colsB, ldB)) return MUON_ERR_CUDA;
    q.epi = reinterpret_cast<const __nv_bfloat16*>(epi);
    q.ld_epi = ld_epi;
    q.out = reinterpret_cast<__nv_bfloat16*>(out);
    q.ld_out = ld_out;
    if (!make_out_map(&q.tmOut, out, M, N, ld_out, op == OP_UPDATE)) return MUON_ERR_CUDA;
    q.M = (int)M;
    q.N = (int)N;
    q.K = (int)K;
    std::vector<NsProblem> pr(1, q);
    rc = upload_phase(np->poly, np->mem.ptr, 0, 256 + sizeof(NsProblem), pr, tiles);
    if (rc) return rc;
    P = np.get();
    ctx->stage_plans[key] = std::move(np);
  }
  NsLaunch L;
  L.nprobs = 1;
  L.deps = nullptr;
  L.ndeps = 0;
  L.pmaps = nullptr;
  L.mirrors = nullptr;
  L.n_mirrors = 0;
  L.mirror_stride = 0;
  L.probs = P->poly.probs;
  L.tiles = P->poly.tiles;
  L.ntiles = P->poly.ntiles;
  L.final_mode = FINAL_NONE;
  L.ca = ca;
  L.cb = cb;
  L.cc = cc;
  L.limit_ns = limit_ns();
  L.status = ctx->status;
  return cuda_err(
      launch_ns_gemm(L, nullptr, pair_grid(ctx, L.ntiles), static_cast<cudaStream_t>(stream), op));
}

static bool ld_ok(long long ld, long long minv) { return ld >= minv && (ld & 7) == 0; }

int muon_gram(const uint16_t* x, int64_t ld_x, uint16_t* a, int64_t ld_a, int64_t m, int64_t n,
              void* stream) {
  if (!x || !a || m <= 0 || n <= 0 || !ld_ok(ld_x, n) || !ld_ok(ld_a, m)) return MUON_ERR_INVALID_ARG;
  if (m >= (1ll << 30) || n >= (1ll << 30)) return MUON_ERR_UNSUPPORTED;
  if (!aligned16(x) || !aligned16(a)) return MUON_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mutex);
  return run_stage(OP_GRAM, x, ld_x, x, ld_x, m, n, nullptr, 0, a, ld_a, m, m, n, 0.f, 0.f, 0.f, stream);
}

int muon_poly(const uint16_t* a, int64_t ld_a, uint16_t* b_out, int64_t ld_b, int64_t m, float cb,
              float cc, void* stream) {
  if (!a || !b_out || m <= 0 || !ld_ok(ld_a, m) || !ld_ok(ld_b, m)) return MUON_ERR_INVALID_ARG;
  if (!std::isfinite(cb) || !std::isfinite(cc)) return MUON_ERR_INVALID_ARG;
  if (m >= (1ll << 30)) return MUON_ERR_UNSUPPORTED;
  if (!aligned16(a) || !aligned16(b_out)) return MUON_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mutex);
  return run_stage(OP_POLY, a, ld_a, a, ld_a, m, m, a, ld_a, b_out, ld_b, m, m, m, 0.f, cb, cc, stream);
}

int muon_xupdate(const uint16_t* b, int64_t ld_b, const uint16_t* x, int64_t ld_x, uint16_t* x_out,
                 int64_t ld_out, int64_t m, int64_t n, float ca, void* stream) {
  if (!b || !x || !x_out || m <= 0 || n <= 0) return MUON_ERR_INVALID_ARG;
  if (!ld_ok(ld_b, m) || !ld_ok(ld_x, n) || !ld_ok(ld_out, n) || !std::isfinite(ca))
    return MUON_ERR_INVALID_ARG;
  if (x_out == x) return MUON_ERR_INVALID_ARG;
  if (m >= (1ll << 30) || n >= (1ll << 30)) return MUON_ERR_UNSUPPORTED;
  if (!aligned16(b) || !aligned16(x) || !aligned16(x_out)) return MUON_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mutex);
  return run_stage(OP_UPDATE, b, ld_b, x, ld_x, m, n, x, ld_x, x_out, ld_out, m, n, m, ca, 0.f, 0.f,
                   stream);
}

int muon_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return MUON_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceCtx* ctx = nullptr;
  int rc = get_ctx(&ctx);
  if (rc) return rc;
  int h = 0;
  if (cudaMemcpy(&h, ctx->status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return MUON_ERR_CUDA;
  if (h != 0 && cudaMemset(ctx->status, 0, sizeof(int)) != cudaSuccess) return MUON_ERR_CUDA;
  return h;
}

const char* muon_error_string(int code) {
  switch (code) {
    case MUON_OK: return "success";
    case MUON_ERR_INVALID_ARG: return "invalid argument";
    case MUON_ERR_UNSUPPORTED: return "unsupported (alignment, size or device)";
    case MUON_ERR_CUDA: return "CUDA error";
    case MUON_ERR_NOMEM: return "out of device memory";
    case MUON_ERR_TIMEOUT: return "device-side wait timed out";
    default: return "unknown status";
  }
}

void muon_set_wait_limit_ns(uint64_t ns) {
  std::lock_guard<std::mutex> lock(g_mutex);
  g_limit_from_env = true;
  g_limit_ns = ns;
}

int64_t muon_workspace_bytes(const int64_t* shapes, int n) {
  if (check_shapes(shapes, n)) return -1;
  int64_t tot = 0;
  for (int g0 = 0; g0 < n; g0 += MUON_MAX_GROUP) {
    const int gn = std::min(MUON_MAX_GROUP, n - g0);
    tot += (int64_t)plan_bytes(make_geom(shapes + 2 * g0, gn), true);
  }
  return tot;
}

int64_t muon_guard_check(void) {
  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceCtx* ctx = nullptr;
  int rc = get_ctx(&ctx);
  if (rc) return rc;
  if (cudaDeviceSynchronize() != cudaSuccess) return MUON_ERR_CUDA;
  int64_t changed = 0;
  unsigned char h[kGuardBytes];
  for (auto& kv : ctx->plans) {
    const Plan& P = *kv.second;
    for (size_t g : P.guards) {
      if (cudaMemcpy(h, P.mem.ptr + g, kGuardBytes, cudaMemcpyDeviceToHost) != cudaSuccess)
        return MUON_ERR_CUDA;
      for (size_t b = 0; b < kGuardBytes; ++b) changed += (h[b] != kGuardByte);
    }
  }
  return changed;
}

void muon_profile_begin(void) {
  std::lock_guard<std::mutex> lock(g_mutex);
  g_prof.on = true;
}

int muon_profile_end(double* ms, int64_t* launches, int nkinds) {
  std::lock_guard<std::mutex> lock(g_mutex);
  g_prof.on = false;
  if (!ms || !launches || nkinds < 0) return MUON_ERR_INVALID_ARG;
  for (int k = 0; k < nkinds; ++k) {
    ms[k] = 0.0;
    launches[k] = 0;
  }
  int rc = MUON_OK;
  for (const ProfRecord& r : g_prof.recs) {
    float t = 0.f;
    if (cudaEventSynchronize(r.stop) != cudaSuccess || cudaEventElapsedTime(&t, r.start, r.stop) != cudaSuccess)
      rc = MUON_ERR_CUDA;
    if (r.kind < nkinds) {
      ms[r.kind] += t;
      launches[r.kind] += 1;
    }
    g_prof.pool.push_back(r.start);
    g_prof.pool.push_back(r.stop);
  }
  g_prof.recs.clear();
  return rc ? rc : std::min(nkinds, (int)MUON_PROFILE_KINDS);
}

void muon_release(void) {
  std::lock_guard<std::mutex> lock(g_mutex);
  int cur = 0;
  cudaGetDevice(&cur);
  for (auto& kv : g_ctx) {
    cudaSetDevice(kv.first);
    cudaDeviceSynchronize();
    kv.second->plans.clear();
    kv.second->stage_plans.clear();
    if (kv.second->status) cudaFree(kv.second->status);
  }
  g_ctx.clear();
  cudaSetDevice(cur);
}

const char* muon_version(void) {
  return kBoundsCheck ? "muon-b200 0.2 (sm_100a, tcgen05, bounds-checked)"
                      : "muon-b200 0.2 (sm_100a, tcgen05)";
}

#ifdef MUON_BOUNDS_CHECK
int muon_debug_set_tile_row(const int64_t* shapes, int n, int ns_steps, int index, int i0) {
  if (check_shapes(shapes, n) || n < 1 || n > MUON_MAX_GROUP) return MUON_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceCtx* ctx = nullptr;
  int rc = get_ctx(&ctx);
  if (rc) return rc;
  auto it = ctx->plans.find(shape_key('S', make_geom(shapes, n)));
  if (it == ctx->plans.end()) return MUON_ERR_INVALID_ARG;
  auto ch = it->second->chains.find(ns_steps);
  if (ch == it->second->chains.end()) return MUON_ERR_INVALID_ARG;
  if (index < 0 || index >= ch->second.ntiles) return MUON_ERR_INVALID_ARG;
  NsTile* tiles = reinterpret_cast<NsTile*>(ch->second.mem->ptr);
  if (cudaDeviceSynchronize() != cudaSuccess) return MUON_ERR_CUDA;
  NsTile t;
  if (cudaMemcpy(&t, tiles + index, sizeof(t), cudaMemcpyDeviceToHost) != cudaSuccess)
    return MUON_ERR_CUDA;
  t.i0 = i0;
  if (cudaMemcpy(tiles + index, &t, sizeof(t), cudaMemcpyHostToDevice) != cudaSuccess)
    return MUON_ERR_CUDA;
  return MUON_OK;
}
#endif

}  // extern "C"
