// internal.h -- data structures shared by the host planner and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "muon.h"

namespace muon {

// Built with -DMUON_BOUNDS_CHECK (newton_schulz_norm_b200.build, checked=True),
// every kernel validates the indices it reads from its tables (tile lists,
// problem and work-item tables) against the sizes it was launched with before
// using them; an invalid entry records MUON_ERR_INVALID_ARG in the status
// word and the work it names is skipped, so a corrupted table becomes an
// error status instead of an access out of bounds.
#ifdef MUON_BOUNDS_CHECK
constexpr bool kBoundsCheck = true;
#else
constexpr bool kBoundsCheck = false;
#endif

// ---------------------------------------------------------------- NS GEMM tiling
// A CTA pair (cluster of 2, tcgen05 cta_group::2) computes a TILE_M x BN
// output tile with M=256, N=256, K=16 MMAs issued by the pair's leader:
// CTA r holds output rows [128 r, 128 r + 128) in its TMEM, A rows
// [128 r, 128 r + 128) and B columns [128 r, 128 r + 128) in its shared
// memory.  Each CTA streams BK-wide K slices through a STAGES-deep ring.
constexpr int BM = 128;                     // output rows per CTA
constexpr int TILE_M = 256;                 // output rows per CTA pair
constexpr int BN = 256;
constexpr int BK = 64;                      // one 128-byte swizzle row of bf16
constexpr int STAGES = 6;                   // every launch but the last update
constexpr int BOX = 64;                     // TMA box: 64 x 64 bf16 = 8 KB
constexpr int BOX_BYTES = BOX * BOX * 2;
constexpr int A_STAGE_BYTES = BM * BK * 2;          // 16 KB: this CTA's rows of A
constexpr int B_STAGE_BYTES = (BN / 2) * BK * 2;    // 16 KB: this CTA's half of B
constexpr int STAGE_BYTES = A_STAGE_BYTES + B_STAGE_BYTES;
constexpr int EPI_WARPS = 8;                // two warps per TMEM lane quarter
constexpr int EPI_THREADS = 32 * EPI_WARPS;
constexpr int GEMM_THREADS = 64 + EPI_THREADS;  // warp 0 TMA, warp 1 MMA, warps 2-9 epilogue
constexpr int TMEM_COLS = 2 * BN;           // two fp32 accumulators of BN columns
constexpr int EPI_LD = 40;                  // padded staging pitch (bf16) of the final kernel
constexpr int EPI_BLOCK_BYTES = 32 * 32 * 2;       // one 32 x 32 bf16 block, 64-byte swizzled
// Per epilogue warp: a block and its mirror (symmetric outputs), or one
// 32 x 64 block with 128-byte swizzle (X update).
constexpr int EPI_STAGE_BYTES = 2 * EPI_BLOCK_BYTES;
constexpr int OUT_BOX = 32;                 // TMA store box: 32 rows x 32 (or 64) bf16
constexpr int GEMM_BAR_BYTES = 512;
constexpr size_t GEMM_SMEM_BYTES =
    size_t(STAGES) * STAGE_BYTES + size_t(EPI_WARPS) * EPI_STAGE_BYTES + 1024 + GEMM_BAR_BYTES;

// The last X update is bound by the fp32 parameter read-modify-write, not by
// the tensor cores, so it trades main-loop stages for a per-warp ring of
// parameter blocks moved by TMA (32 x 32 fp32, 128-byte swizzle).
constexpr int FINAL_STAGES = 3;             // the last update with mirrors (parameter ring)
constexpr int P_RING = 4;                    // parameter blocks per epilogue warp
constexpr int P_AHEAD = P_RING - 2;          // chunks whose blocks are loaded ahead
constexpr int E_AHEAD = 1;                   // chunks whose a*X input is loaded ahead
constexpr int P_BLOCK_BYTES = 32 * 32 * 4;
constexpr int FINAL_EPI_BYTES = P_RING * P_BLOCK_BYTES;   // per epilogue warp
constexpr size_t FINAL_SMEM_BYTES =
    size_t(FINAL_STAGES) * STAGE_BYTES + size_t(EPI_WARPS) * FINAL_EPI_BYTES + 1024 + GEMM_BAR_BYTES;
// The last update without mirrors reads no parameters: two increment blocks
// per epilogue warp, and the space left over goes to main-loop stages.
constexpr int REDUCE_STAGES = 4;
constexpr int REDUCE_EPI_BYTES = 2 * P_BLOCK_BYTES;
constexpr size_t REDUCE_SMEM_BYTES =
    size_t(REDUCE_STAGES) * STAGE_BYTES + size_t(EPI_WARPS) * REDUCE_EPI_BYTES + 1024 + GEMM_BAR_BYTES;

enum NsOp : int { OP_GRAM = 0, OP_POLY = 1, OP_UPDATE = 2 };

// What the X-update epilogue does with X_{k+1}.
enum FinalMode : int {
  FINAL_NONE = 0,      // store bf16 X_{k+1} to the next iterate buffer
  FINAL_PARAM = 1,     // p <- p - scale * X_{k+1}   (fp32, stored orientation)
  FINAL_OUT_F32 = 2,   // out <- X_{k+1} as fp32     (stored orientation)
  FINAL_OUT_BF16 = 3,  // out <- X_{k+1} as bf16     (stored orientation)
};

// One matrix of one GEMM phase.  Lives in device memory; 64-byte aligned
// because the tensor maps inside are read by TMA from global memory.
struct alignas(64) NsProblem {
  CUtensorMap tmA;            // A operand source: K-major rows x K
  CUtensorMap tmB;            // B operand source: K-major (Gram, poly) or MN-major (update)
  CUtensorMap tmOut;          // bf16 output, 32 x 32 boxes, 64-byte swizzle (TMA stores)
  const __nv_bfloat16* epi;   // poly: A (for b*A); update: X (for a*X)
  __nv_bfloat16* out;         // bf16 output (A, B or X_{k+1})
  long long ld_epi;
  long long ld_out;
  int M, N, K;                // output M x N, reduction length K
  int transposed;             // final modes: output (i, j) lands at [j][i]
  long long ld_final;         // leading dimension of the final target
  int slot;                   // index into FinalTable
  int pad_[3];
};

struct NsTile {
  int prob;       // index into the NsProblem array
  int i0;         // first output row
  int j0;         // first output column
  int kc;         // number of BK slices
  int op;         // NsOp of this tile
  int wait_idx;   // chain launch: counter (in NsLaunch::deps) to wait for, or -1
  int wait_need;  //   ... until it reaches this value (16 per tile of the phase before)
  int done_idx;   // chain launch: counter to count this tile's stores in, or -1
};

struct FinalTable {
  void* ptr[MUON_MAX_GROUP];
  float scale[MUON_MAX_GROUP];
};

struct NsLaunch {
  const NsProblem* probs;
  const NsTile* tiles;
  int ntiles;
  int nprobs;                // entries of probs (checked builds validate tile.prob)
  // Chain launches: one completion counter per (phase, matrix), zeroed before
  // the launch; tiles name them by index (checked builds validate < ndeps).
  int* deps;
  int ndeps;
  int final_mode;
  // Final FINAL_PARAM launch only: one tensor map per matrix (indexed by
  // NsProblem::slot) over the stored fp32 parameters, 32 x 32 boxes with
  // 128-byte swizzle; nullptr selects the register read-modify-write path.
  const CUtensorMap* pmaps;
  // Final FINAL_PARAM launch with mirrors only: a device array of
  // n_mirrors x mirror_stride parameter pointers; entry k * mirror_stride +
  // slot receives a copy of every updated block of matrix `slot` (the same
  // layout as the parameter; the pointer may be another GPU's memory).
  float* const* mirrors;
  int n_mirrors;
  int mirror_stride;
  float ca, cb, cc;
  unsigned long long limit_ns;
  int* status;
};

// ---------------------------------------------------------------- fused first kernel
// Momentum + Nesterov + Frobenius norm + bf16 cast + orientation, over
// 64 x 64 tiles of the stored matrix, in two passes joined per matrix.
constexpr int K1_TILE = 64;
constexpr int K1_THREADS = 256;
constexpr int K1_GROUP = 4;  // 64x64 tiles per work item (one norm partial, one fence)

enum K1Mode : int { K1_MOMENTUM = 0, K1_PLAIN = 1 };

struct K1Info {              // static per matrix (device memory)
  long long r, c;            // stored shape
  long long ldx;             // leading dimension of the oriented bf16 X0
  int tiles_c;               // tiles along the stored columns
  int ntiles;                // tiles of this matrix
  int nitems;                // work items of this matrix (groups of K1_GROUP tiles)
  int part0;                 // offset of its partial sums (one per item)
  int transposed;            // r > c
};

struct K1Ptrs {              // per call
  const float* g;            // gradient (or the matrix to orthogonalise)
  float* buf;                // momentum buffer (unused in K1_PLAIN)
  __nv_bfloat16* x0;         // oriented bf16 output
};

// Work item: a matrix (K1_PASS2 set for its second pass) and a group of
// K1_GROUP consecutive tiles of it.
struct K1Item {
  int mat;                   // matrix index; pass 2 items have mat | 0x40000000
  int group;                 // tiles [group * K1_GROUP, +K1_GROUP) of the matrix
};
constexpr int K1_PASS2 = 0x40000000;

struct K1Launch {
  const K1Info* info;
  const K1Item* items;
  int nitems;
  int n;                     // matrices (entries of info and ptrs)
  int npartials;             // entries of partials
  int mode;
  int nesterov;
  float beta;
  int* counter;              // work-queue head (zeroed before launch)
  int* done;                 // [n] pass-1 tiles finished (zeroed)
  int* ready;                // [n] norm published (zeroed)
  double* partials;          // per tile sum of squares
  double* norms;             // [n] Frobenius norms
  unsigned long long limit_ns;
  int* status;
  K1Ptrs ptrs[MUON_MAX_GROUP];
};

// Applies p <- p - scale * X0 when ns_steps == 0 (no GEMM epilogue to fuse into).
struct ApplyLaunch {
  const K1Info* info;
  int n;
  int mode;                  // FINAL_PARAM / FINAL_OUT_F32 / FINAL_OUT_BF16
  K1Ptrs ptrs[MUON_MAX_GROUP];   // x0 = source, g unused
  void* dst[MUON_MAX_GROUP];
  float scale[MUON_MAX_GROUP];
};

// ---------------------------------------------------------------- AdamW
// One AdamW step over a list of fp32 tensors of any size: the parameters the
// Muon step leaves out.  Each tensor is cut into chunks of ADAMW_CHUNK
// elements; persistent CTAs take chunks in grid-stride order.
constexpr int ADAMW_THREADS = 256;
constexpr int ADAMW_VEC = 2;                                   // float4 per array per thread
constexpr int ADAMW_CHUNK = ADAMW_THREADS * ADAMW_VEC * 4;     // 2048 elements
constexpr int ADAMW_MAX_TENSORS = 128;                         // per launch

struct AdamWTensor {
  float* p;
  const float* g;
  float* m;                  // running average of the gradient
  float* v;                  // running average of its square
  long long numel;           // > 0
  int chunk0;                // first chunk of this tensor in the launch
  int vec;                   // all four pointers 16-byte aligned: float4 path
  float decay;               // fp32(1 - lr * weight_decay_i)
  int pad_;
};

struct AdamWLaunch {
  int n;                     // tensors in this launch
  int nchunks;               // chunks of all of them
  float beta1, one_minus_beta1;
  float beta2, one_minus_beta2;
  float step_size;           // fp32(lr / (1 - beta1^t))
  float inv_sqrt_bc2;        // fp32(1 / sqrt(1 - beta2^t))
  float eps;
  AdamWTensor t[ADAMW_MAX_TENSORS];
};

// ---------------------------------------------------------------- launchers
// op: the NsOp of every tile of the launch, or -1 for a chain launch.
cudaError_t launch_ns_gemm(const NsLaunch& L, const FinalTable* F, int grid, cudaStream_t stream,
                           int op);
cudaError_t ns_gemm_setup(int device);
int ns_gemm_max_pairs();
cudaError_t launch_k1(const K1Launch& L, int grid, cudaStream_t stream);
int k1_blocks_per_sm();
cudaError_t launch_apply(const ApplyLaunch& L, cudaStream_t stream);
cudaError_t launch_adamw(const AdamWLaunch& L, int grid, cudaStream_t stream);
int adamw_blocks_per_sm();
// The bound of every device-side wait, in ns (muon_set_wait_limit_ns, else
// MUON_SPIN_LIMIT_NS at first use, else 2 s).  Takes the interface's lock.
unsigned long long current_wait_limit_ns();

}  // namespace muon
