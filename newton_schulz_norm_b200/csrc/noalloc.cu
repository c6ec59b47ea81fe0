// noalloc.cu -- muon_momentum_normalize_noalloc: the fused first kernel
// (momentum, Nesterov, Frobenius norm, bf16 cast, orientation) without any
// memory allocation.
//
// Who needs it: callers that cannot call cudaMalloc at the time they run the
// optimizer -- a host that has handed all device memory to its own pool
// allocator, a process that must not grow its footprint after start-up, or
// code running where allocation is not allowed.  The regular entry point
// allocates its scratch (work queue, counters, norm partials) on first use;
// this one keeps that scratch in a fixed-size array compiled into the library
// instead.  The caller still passes every input and output.
//
// The scratch array below is a file-scope __device__ array: every GPU that
// loads this library holds it (about 200 KB) until the process exits.  In
// host code its name is only a host-side stand-in, not a device address, so
// the address handed to the kernels comes from cudaGetSymbolAddress, taken
// once per device (with that device current) on the first call.  That first
// call on a device therefore does the set-up and should come before any
// stream capture.
//
// Every call shares the one array and it keeps the last call's contents: the
// set-up kernel clears what must start at zero (queue head, per-matrix
// counters and flags) at the start of every call.  Calls whose executions
// overlap on the GPU (different streams, or different host threads without
// ordering) race on the array; order them on one stream.
#include <algorithm>
#include <cmath>
#include <mutex>

#include "internal.h"
#include "ptx.cuh"

namespace muon {
namespace {

constexpr int kMaxMats = MUON_NOALLOC_MAX_MATRICES;
constexpr int kMaxItems = MUON_NOALLOC_MAX_ITEMS;   // pass-1 and pass-2 items together
constexpr int kMaxDevices = 64;

struct NoAllocScratch {
  int counters[1 + 2 * kMaxMats];   // queue head, done[kMaxMats], ready[kMaxMats]
  int status;                       // timeouts land here when no status word is given
  double norms[kMaxMats];
  double partials[kMaxItems / 2];   // one per pass-1 item
  K1Info info[kMaxMats];
  K1Item items[kMaxItems];
};

static __device__ __align__(256) unsigned char g_noalloc_scratch[sizeof(NoAllocScratch)];

struct SetupArgs {
  int n;
  int nitems;                       // total work items (both passes)
  long long slack;                  // pass-1 items queued before a matrix's pass 2
  K1Info info[kMaxMats];
};

// Writes the per-matrix table and the work queue, in the regular entry
// point's order (a matrix's pass-2 items follow `slack` further pass-1 items,
// inserted between single pass-1 items), and clears the counters.  The queue
// is a list of runs: run s covers queue positions [seg_start[s],
// seg_start[s+1]) and holds items seg_first[s], ... of matrix seg_mat[s].
// Runs on the caller's stream before the kernel.
constexpr int kMaxRuns = 3 * kMaxMats;   // a pass-2 run can split a pass-1 run in two

__global__ void noalloc_setup_kernel(const __grid_constant__ SetupArgs S, NoAllocScratch* scr) {
  __shared__ int seg_start[kMaxRuns + 1];
  __shared__ int seg_mat[kMaxRuns];
  __shared__ int seg_first[kMaxRuns];
  __shared__ int nseg;
  if (threadIdx.x == 0) {
    int k = 0, at = 0;
    auto add = [&](int mat, int first, int count) {
      if (count <= 0) return;
      seg_start[k] = at;
      seg_mat[k] = mat;
      seg_first[k] = first;
      at += count;
      ++k;
    };
    long long end1[kMaxMats];
    long long queued = 0;
    int next2 = 0;
    for (int i = 0; i < S.n; ++i) {
      const int ni = S.info[i].nitems;
      int run0 = 0;                  // first pass-1 item of i not yet in a run
      for (int t = 0; t < ni; ++t) {
        ++queued;
        if (next2 < i && queued - end1[next2] >= S.slack) {
          add(i, run0, t + 1 - run0);   // pass-1 items run0 .. t
          run0 = t + 1;
          while (next2 < i && queued - end1[next2] >= S.slack) {
            add(next2 | K1_PASS2, 0, S.info[next2].nitems);
            ++next2;
          }
        }
      }
      add(i, run0, ni - run0);
      end1[i] = queued;
    }
    while (next2 < S.n) {
      add(next2 | K1_PASS2, 0, S.info[next2].nitems);
      ++next2;
    }
    seg_start[k] = at;
    nseg = k;
  }
  __syncthreads();
  if (blockIdx.x == 0) {
    for (int t = threadIdx.x; t < 1 + 2 * kMaxMats; t += blockDim.x) scr->counters[t] = 0;
    for (int t = threadIdx.x; t < S.n; t += blockDim.x) scr->info[t] = S.info[t];
    if (threadIdx.x == 0) scr->status = 0;
  }
  for (int it = blockIdx.x * blockDim.x + threadIdx.x; it < S.nitems; it += gridDim.x * blockDim.x) {
    int s = 0;
    while (s + 1 < nseg && seg_start[s + 1] <= it) ++s;
    K1Item item;
    item.mat = seg_mat[s];
    item.group = seg_first[s] + (it - seg_start[s]);
    scr->items[it] = item;
  }
}

std::mutex g_noalloc_mutex;
void* g_scratch_addr[kMaxDevices] = {};
int g_num_sms[kMaxDevices] = {};
int g_blocks_per_sm[kMaxDevices] = {};

long long cdiv_ll(long long a, long long b) { return (a + b - 1) / b; }

// Once per device: check the architecture and take the array's device address.
int noalloc_device_setup(int dev, NoAllocScratch** scr, int* sms, int* bps) {
  if (dev < 0 || dev >= kMaxDevices) return MUON_ERR_UNSUPPORTED;
  if (!g_scratch_addr[dev]) {
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return MUON_ERR_CUDA;
    if (prop.major != 10) return MUON_ERR_UNSUPPORTED;   // built for sm_100a only
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return MUON_ERR_CUDA;
    g_num_sms[dev] = prop.multiProcessorCount;
    g_blocks_per_sm[dev] = k1_blocks_per_sm();
    g_scratch_addr[dev] = p;
  }
  *scr = static_cast<NoAllocScratch*>(g_scratch_addr[dev]);
  *sms = g_num_sms[dev];
  *bps = g_blocks_per_sm[dev];
  return MUON_OK;
}

bool aligned16_na(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace muon

using namespace muon;

extern "C" int muon_momentum_normalize_noalloc(const float* const* grads, float* const* bufs,
                                               uint16_t* const* x0, const int64_t* x0_ld,
                                               const int64_t* shapes, int n, float beta,
                                               int nesterov, int* dev_status, void* stream) {
  if (n < 0) return MUON_ERR_INVALID_ARG;
  if (n == 0) return MUON_OK;
  if (n > kMaxMats) return MUON_ERR_UNSUPPORTED;   // beyond the fixed scratch
  if (!grads || !bufs || !x0 || !x0_ld || !shapes || !std::isfinite(beta)) return MUON_ERR_INVALID_ARG;
  if (dev_status && (reinterpret_cast<uintptr_t>(dev_status) & 3u)) return MUON_ERR_UNSUPPORTED;
  static thread_local SetupArgs S;
  long long items = 0;
  for (int i = 0; i < n; ++i) {
    const long long r = shapes[2 * i], c = shapes[2 * i + 1];
    if (r <= 0 || c <= 0) return MUON_ERR_INVALID_ARG;
    if (r * c >= (1ll << 31) || r >= (1ll << 30) || c >= (1ll << 30)) return MUON_ERR_UNSUPPORTED;
    if (!grads[i] || !bufs[i] || !x0[i]) return MUON_ERR_INVALID_ARG;
    if (!aligned16_na(grads[i]) || !aligned16_na(bufs[i]) || !aligned16_na(x0[i]))
      return MUON_ERR_UNSUPPORTED;
    const long long ncols = r > c ? r : c;
    if (x0_ld[i] < ncols || (x0_ld[i] & 7)) return MUON_ERR_INVALID_ARG;
    K1Info& k = S.info[i];
    k.r = r;
    k.c = c;
    k.ldx = x0_ld[i];
    k.tiles_c = (int)cdiv_ll(c, K1_TILE);
    k.ntiles = (int)(cdiv_ll(r, K1_TILE) * k.tiles_c);
    k.nitems = (int)cdiv_ll(k.ntiles, K1_GROUP);
    k.part0 = (int)items;
    k.transposed = r > c;
    items += k.nitems;
    if (2 * items > kMaxItems) return MUON_ERR_UNSUPPORTED;   // beyond the fixed scratch
  }
  S.n = n;
  S.nitems = (int)(2 * items);
  const unsigned long long limit = current_wait_limit_ns();   // before this file's own lock

  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MUON_ERR_CUDA;
  NoAllocScratch* scr = nullptr;
  int sms = 0, bps = 0;
  int rc = noalloc_device_setup(dev, &scr, &sms, &bps);
  if (rc) return rc;

  S.slack = std::max(1, sms * bps / 2);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int setup_grid = (int)std::min<long long>(64, cdiv_ll(S.nitems, 256));
  noalloc_setup_kernel<<<setup_grid, 256, 0, s>>>(S, scr);
  if (cudaGetLastError() != cudaSuccess) return MUON_ERR_CUDA;

  static thread_local K1Launch L;
  L.info = scr->info;
  L.items = scr->items;
  L.nitems = S.nitems;
  L.n = n;
  L.npartials = kMaxItems / 2;
  L.mode = K1_MOMENTUM;
  L.nesterov = nesterov;
  L.beta = beta;
  L.counter = scr->counters;
  L.done = scr->counters + 1;
  L.ready = scr->counters + 1 + n;
  L.partials = scr->partials;
  L.norms = scr->norms;
  L.limit_ns = limit;
  L.status = dev_status ? dev_status : &scr->status;
  for (int i = 0; i < n; ++i) {
    L.ptrs[i].g = grads[i];
    L.ptrs[i].buf = bufs[i];
    L.ptrs[i].x0 = reinterpret_cast<__nv_bfloat16*>(x0[i]);
  }
  const int grid = std::max(1, std::min(S.nitems, sms * bps));
  return launch_k1(L, grid, s) == cudaSuccess ? MUON_OK : MUON_ERR_CUDA;
}
