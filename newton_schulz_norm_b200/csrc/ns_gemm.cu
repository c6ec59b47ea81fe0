// ns_gemm.cu -- the three tensor-core products of one quintic Newton-Schulz
// iteration on sm_100a:
//
//   OP_GRAM    A  = bf16(X X^T)              upper-triangle tiles, mirrored
//   OP_POLY    B  = bf16(b A + c A A^T)      A symmetric, so A A = A A^T
//   OP_UPDATE  X' = bf16(a X + B X)          optionally fused with the update
//                                            p <- p - lr*s*X' on the last step
//
// (X thread on the new NanoGPT optimizer, tweets 5/8 and 6/8: quintic
// Newton-Schulz, in bfloat16.)
//
// Design: a persistent, warp-specialised kernel per phase that runs every
// matrix of the phase as one grouped launch.  CTAs work in pairs (clusters
// of two on neighbouring SMs, tcgen05 cta_group::2) on 256 x 256 output
// tiles; CTA r of a pair holds rows [128r, 128r+128) of the A operand and
// columns [128r, 128r+128) of the B operand.  Per CTA:
//   warp 0     one thread issues TMA tile loads (64x64 bf16 boxes, 128-byte
//              swizzle, no multicast) into a ring of shared-memory stages;
//              both CTAs' bytes complete on the leader CTA's barrier;
//   warp 1     (leader only) one thread issues tcgen05.mma.cta_group::2
//              (M=256, N=256, K=16, fp32 accumulation in TMEM) and commits
//              stages back to both CTAs' rings;
//   warps 2-9  the epilogue: two warps per TMEM lane quarter, each taking
//              four 32-column chunks of its 32 rows.  A warp reads its chunk
//              from TMEM (tcgen05.ld, one row per thread), combines it with
//              the epilogue input (fetched before the accumulator is ready;
//              in the polynomial launch read from operand slices held in
//              the ring, see hold_range), writes bf16 rows into a swizzled
//              staging block and stores it with a TMA store: 32 x 32 blocks
//              for symmetric outputs, which store each block above the
//              diagonal twice (as itself and mirrored); 32 x 64 blocks, two
//              chunks per store, for the X update.
// Two TMEM accumulators (2 x 256 columns) let the epilogue of one tile
// overlap the main loop of the next.  The last update adds its fp32
// parameter increments with TMA reduce-adds instead (or, when mirrors need
// the final values, moves the parameter blocks through a per-warp ring of TMA
// loads and stores).
//
// Every tile carries its operation, so one launch can run several phases:
// the chain launch runs every Gram, polynomial and X-update tile of all
// iterations but the last update, in phase order.  A tile of phase q of
// matrix i waits (producer: before its first operand load; epilogue: before
// reading its input) until every tile of phase q-1 of matrix i has been
// stored, which the epilogue warps count in a per-(phase, matrix) counter
// after their stores complete (release / acquire at GPU scope, with a proxy
// fence on both sides since the stores and loads are TMA's).  Within one
// launch a matrix's phases thus follow one another, while other matrices'
// tiles fill the GPU, instead of a launch boundary and a full drain between
// phases.  Every wait is bounded.
#include <cstdio>

#include "internal.h"
#include "ptx.cuh"

namespace muon {

namespace {

// Waits that only drain this CTA's own in-flight copies or MMAs before it
// exits use a fixed bound, independent of the caller's wait limit, so that
// even a limit of 0 never lets a CTA leave with work still landing in its
// shared memory or TMEM.
constexpr unsigned long long kDrainLimitNs = 1000000000ull;

constexpr uint32_t kIdescK = idesc_bf16_f32(TILE_M, BN, 0);   // pair MMA, B K-major
constexpr uint32_t kIdescMN = idesc_bf16_f32(TILE_M, BN, 1);  // pair MMA, B MN-major
constexpr int HOLD_CHUNKS = BN / BK;                       // K slices of one 256-wide block: 4
constexpr int CHUNKS_PER_WARP = BN / 32 / 2;               // 4

__device__ __forceinline__ void record_status(int* status, int code) {
  atomicCAS(status, 0, code);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ void unpack8(const uint4& w, float* o) {
  const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    o[2 * t] = bf16_bits_to_float(u[t] & 0xFFFFu);
    o[2 * t + 1] = bf16_bits_to_float(u[t] >> 16);
  }
}

__device__ __forceinline__ uint4 pack8(const float* x) {
  uint4 w;
  w.x = pack_bf16x2(x[0], x[1]);
  w.y = pack_bf16x2(x[2], x[3]);
  w.z = pack_bf16x2(x[4], x[5]);
  w.w = pack_bf16x2(x[6], x[7]);
  return w;
}

// This lane's row of the epilogue input: 32 bf16 at (row, col0 .. col0+31)
// as four 16-byte loads (zeros outside the matrix).
// The chain launch reads inputs that other CTAs of the same launch wrote, so
// it may not use the non-coherent (read-only) path that one-phase launches
// use for inputs of an earlier launch: its loads are plain
// weak ld.global, which the GPU-scope acquire that precedes them orders after
// the writers' release (L1 lines included).  Such loads still allocate in
// L1, which matters: each lane reads 64 contiguous bytes in four 16-byte
// loads, and L2-only loads cost every X update about 85 us on GPT-2 124M.
__device__ __forceinline__ uint4 ld_global_weak(const void* p) {
  uint4 v;
  asm volatile("ld.global.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p)
               : "memory");
  return v;
}

__device__ __forceinline__ unsigned short ld_global_weak_u16(const void* p) {
  unsigned short v;
  asm volatile("ld.global.u16 %0, [%1];" : "=h"(v) : "l"(p) : "memory");
  return v;
}

template <bool COHERENT = false>
__device__ __forceinline__ void load_row(const __nv_bfloat16* src, long long ld, int row, int col0,
                                         int M, int N, uint4 (&r)[4]) {
  const __nv_bfloat16* p = src + (long long)row * ld + col0;
  if (row < M && col0 + 32 <= N) {
#pragma unroll
    for (int q = 0; q < 4; ++q)
      r[q] = COHERENT ? ld_global_weak(reinterpret_cast<const uint4*>(p) + q)
                      : __ldg(reinterpret_cast<const uint4*>(p) + q);
    return;
  }
  uint16_t h[32];
#pragma unroll
  for (int e = 0; e < 32; ++e)
    h[e] = (row < M && col0 + e < N)
               ? (COHERENT ? ld_global_weak_u16(p + e) : __bfloat16_as_ushort(p[e]))
               : 0;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    r[q].x = h[8 * q + 0] | ((uint32_t)h[8 * q + 1] << 16);
    r[q].y = h[8 * q + 2] | ((uint32_t)h[8 * q + 3] << 16);
    r[q].z = h[8 * q + 4] | ((uint32_t)h[8 * q + 5] << 16);
    r[q].w = h[8 * q + 6] | ((uint32_t)h[8 * q + 7] << 16);
  }
}

// A 32 x 32 bf16 staging block in the TMA 64-byte-swizzle layout: row r
// occupies bytes [64 r, 64 r + 64) and its 16-byte chunk q sits at chunk
// position q ^ ((r >> 1) & 3).  Row-per-lane writes are bank-conflict free.
__device__ __forceinline__ uint32_t sw64(int r, int q) {
  return (uint32_t)(r * 64 + ((q ^ ((r >> 1) & 3)) << 4));
}

__device__ __forceinline__ void row_to_block(uint8_t* blk, int lane, const float (&x)[32]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) *reinterpret_cast<uint4*>(blk + sw64(lane, q)) = pack8(x + 8 * q);
}

// The lane's 32 values become column `lane` of the block (the mirror image).
__device__ __forceinline__ void col_to_block(uint8_t* blk, int lane, const float (&x)[32]) {
  const int q = lane >> 3, e = lane & 7;
#pragma unroll
  for (int c = 0; c < 32; ++c)
    *reinterpret_cast<uint16_t*>(blk + sw64(c, q) + 2 * e) =
        __bfloat16_as_ushort(__float2bfloat16_rn(x[c]));
}

// Chunk `second` (0 or 1) of a 32 x 64 bf16 staging block in the TMA 128-byte
// swizzle (row r: bytes [128 r, 128 r + 128), 16-byte unit u at u ^ (r & 7)):
// the lane's row, columns 32 second .. 32 second + 31.  Bank-conflict free.
__device__ __forceinline__ void row_to_wide(uint8_t* blk, int lane, int second, const float (&x)[32]) {
#pragma unroll
  for (int q = 0; q < 4; ++q)
    *reinterpret_cast<uint4*>(blk + lane * 128 + (((4 * second + q) ^ (lane & 7)) << 4)) =
        pack8(x + 8 * q);
}

// Diagonal block: entries below the diagonal take the value computed above
// it, so the stored block is exactly symmetric.  Reads touch only entries
// above the diagonal and writes only entries below it.
__device__ __forceinline__ void symmetrize_block(uint8_t* blk, int lane) {
  const int r = lane;
#pragma unroll
  for (int c = 0; c < 32; ++c) {
    if (c < r) {
      const uint16_t v = *reinterpret_cast<const uint16_t*>(blk + sw64(c, r >> 3) + 2 * (r & 7));
      *reinterpret_cast<uint16_t*>(blk + sw64(r, c >> 3) + 2 * (c & 7)) = v;
    }
  }
}

// This lane's 32 epilogue inputs from a held operand slice (see hold_range):
// row rr of this CTA's A rows, K values k0 .. k0+31.  The slice holds two
// TMA boxes of 64 rows x 128 bytes in the 128-byte swizzle: 16-byte unit u
// of row r sits at unit u ^ (r & 7).
__device__ __forceinline__ void held_row(const uint8_t* sa, int rr, int k0, uint4 (&e)[4]) {
  const uint8_t* rowp = sa + (rr >> 6) * BOX_BYTES + (rr & 63) * 128;
  const int sw = rr & 7;
#pragma unroll
  for (int v = 0; v < 4; ++v)
    e[v] = *reinterpret_cast<const uint4*>(rowp + ((((k0 >> 3) + v) ^ sw) << 4));
}

// One bf16 row per lane -> staging block (row-major).
__device__ __forceinline__ void rows_to_stage(uint16_t* stg, const float (&x)[32], int lane) {
#pragma unroll
  for (int q = 0; q < 4; ++q)
    *reinterpret_cast<uint4*>(stg + lane * EPI_LD + q * 8) = pack8(x + 8 * q);
  __syncwarp();
}

// Staging block -> global, coalesced.  Element (r, c) of the block goes to
// dst[(rbase + r) * ld + col0 + c] when (rbase + r) < M, (col0 + c) < N and,
// for triangle stores, col0 + c >= rbase + r + tri_shift (tri_shift = 0: on
// or above the diagonal; 1: strictly above; -1 disables the test).
__device__ __forceinline__ void stage_to_global(const uint16_t* stg, __nv_bfloat16* dst, long long ld,
                                                int rbase, int col0, int M, int N, int lane,
                                                int tri_shift) {
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int r = (lane >> 2) + 8 * k;
    const int c = (lane & 3) * 8;
    const int grow = rbase + r, gcol = col0 + c;
    if (grow >= M || gcol >= N) continue;
    const uint4 w = *reinterpret_cast<const uint4*>(stg + r * EPI_LD + c);
    __nv_bfloat16* p = dst + (long long)grow * ld + gcol;
    const bool full = (gcol + 8 <= N) && (tri_shift < 0 || gcol >= grow + tri_shift);
    if (full) {
      *reinterpret_cast<uint4*>(p) = w;
    } else {
      const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const bool ok = (gcol + e < N) && (tri_shift < 0 || gcol + e >= grow + tri_shift);
        if (ok) p[e] = __ushort_as_bfloat16((uint16_t)((u[e >> 1] >> (16 * (e & 1))) & 0xFFFFu));
      }
    }
  }
  __syncwarp();
}

// The final iteration's output: X (bf16-rounded) applied to, or written
// into, the caller's buffer in the stored orientation.  The parameter block a
// lane needs is fetched by final_load one chunk ahead of final_apply, so the
// fp32 read-modify-write of one chunk overlaps the reads of the next.
//
// Lane layout of the 32x32 block: transposed targets (X(row, col) at
// [col][row]) use lane = row, value c = column (each column one coalesced
// 128-byte segment); other targets use lane -> rows (lane>>3) + 4k,
// columns (lane&7)*4 .. +3 (4 rows x 128 contiguous bytes per instruction).
__device__ __forceinline__ void final_load(const NsProblem& P, const FinalTable* F, int mode,
                                           int rbase, int col0, int lane, float (&pv)[32]) {
  if (mode != FINAL_PARAM) return;
  const int M = P.M, N = P.N;
  const long long ldf = P.ld_final;
  const float* base = reinterpret_cast<const float*>(F->ptr[P.slot]);
  if (P.transposed) {
    const int row = rbase + lane;
    const bool rok = row < M;
#pragma unroll
    for (int c = 0; c < 32; ++c)
      pv[c] = (rok && col0 + c < N) ? base[(long long)(col0 + c) * ldf + row] : 0.f;
    return;
  }
  const bool vec_ok = (ldf & 3) == 0;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const int grow = rbase + (lane >> 3) + 4 * k, gcol = col0 + (lane & 7) * 4;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (grow < M && gcol < N) {
      const float* q = base + (long long)grow * ldf + gcol;
      if (vec_ok && gcol + 4 <= N) {
        v = *reinterpret_cast<const float4*>(q);
      } else {
        v.x = q[0];
        if (gcol + 1 < N) v.y = q[1];
        if (gcol + 2 < N) v.z = q[2];
        if (gcol + 3 < N) v.w = q[3];
      }
    }
    pv[4 * k + 0] = v.x;
    pv[4 * k + 1] = v.y;
    pv[4 * k + 2] = v.z;
    pv[4 * k + 3] = v.w;
  }
}

__device__ __forceinline__ void final_apply(const NsProblem& P, const FinalTable* F, int mode,
                                            uint16_t* stg, const float (&xb)[32], int rbase,
                                            int col0, int lane, const float (&pv)[32]) {
  const int M = P.M, N = P.N;
  const int slot = P.slot;
  const long long ldf = P.ld_final;
  const float neg_scale = -F->scale[slot];
  if (P.transposed) {
    const int row = rbase + lane;
    const bool rok = row < M;
    if (mode == FINAL_PARAM) {
      float* base = reinterpret_cast<float*>(F->ptr[slot]);
#pragma unroll
      for (int c = 0; c < 32; ++c)
        if (rok && col0 + c < N)
          base[(long long)(col0 + c) * ldf + row] = __fadd_rn(pv[c], __fmul_rn(neg_scale, xb[c]));
    } else if (mode == FINAL_OUT_F32) {
      float* base = reinterpret_cast<float*>(F->ptr[slot]);
#pragma unroll
      for (int c = 0; c < 32; ++c)
        if (rok && col0 + c < N) base[(long long)(col0 + c) * ldf + row] = xb[c];
    } else {
      __nv_bfloat16* base = reinterpret_cast<__nv_bfloat16*>(F->ptr[slot]);
#pragma unroll
      for (int c = 0; c < 32; ++c)
        if (rok && col0 + c < N) base[(long long)(col0 + c) * ldf + row] = __float2bfloat16_rn(xb[c]);
    }
    return;
  }
  rows_to_stage(stg, xb, lane);
  if (mode == FINAL_OUT_BF16) {
    stage_to_global(stg, reinterpret_cast<__nv_bfloat16*>(F->ptr[slot]), ldf, rbase, col0, M, N,
                    lane, -1);
    return;
  }
  float* base = reinterpret_cast<float*>(F->ptr[slot]);
  const bool vec_ok = (ldf & 3) == 0;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const int r = (lane >> 3) + 4 * k, c = (lane & 7) * 4;
    const int grow = rbase + r, gcol = col0 + c;
    if (grow >= M || gcol >= N) continue;
    const uint2 w = *reinterpret_cast<const uint2*>(stg + r * EPI_LD + c);
    const float x4[4] = {bf16_bits_to_float(w.x & 0xFFFFu), bf16_bits_to_float(w.x >> 16),
                         bf16_bits_to_float(w.y & 0xFFFFu), bf16_bits_to_float(w.y >> 16)};
    float4 o;
    if (mode == FINAL_PARAM) {
      o.x = __fadd_rn(pv[4 * k + 0], __fmul_rn(neg_scale, x4[0]));
      o.y = __fadd_rn(pv[4 * k + 1], __fmul_rn(neg_scale, x4[1]));
      o.z = __fadd_rn(pv[4 * k + 2], __fmul_rn(neg_scale, x4[2]));
      o.w = __fadd_rn(pv[4 * k + 3], __fmul_rn(neg_scale, x4[3]));
    } else {
      o = make_float4(x4[0], x4[1], x4[2], x4[3]);
    }
    float* q = base + (long long)grow * ldf + gcol;
    if (vec_ok && gcol + 4 <= N) {
      *reinterpret_cast<float4*>(q) = o;
    } else {
      q[0] = o.x;
      if (gcol + 1 < N) q[1] = o.y;
      if (gcol + 2 < N) q[2] = o.z;
      if (gcol + 3 < N) q[3] = o.w;
    }
  }
  __syncwarp();
}

// Copies one finished 32 x 32 fp32 parameter block (128-byte swizzle: block
// element (r, c) at r*128 + (((c >> 2) ^ (r & 7)) << 4) + (c & 3)*4) from
// shared memory to every mirror of its matrix.  Block element (r, c) is
// parameter element (base_r + r, base_c + c).  Each store instruction of the
// warp writes four whole 128-byte rows: lane l takes 16-byte chunk l & 7 of
// rows (l >> 3) + 4k.
__device__ __forceinline__ void mirror_block(const NsLaunch& L, const NsProblem& P,
                                             const uint8_t* blk, int base_r, int base_c, int lane) {
  const int R = P.transposed ? P.N : P.M;   // parameter rows and columns
  const int C = P.transposed ? P.M : P.N;
  const int q = lane & 7;
  const int col = base_c + 4 * q;
  float4 v[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const int r = (lane >> 3) + 4 * k;
    v[k] = *reinterpret_cast<const float4*>(blk + r * 128 + ((q ^ (r & 7)) << 4));
  }
  if (col >= C) return;
  for (int m = 0; m < L.n_mirrors; ++m) {
    float* dst = L.mirrors[m * L.mirror_stride + P.slot];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int prow = base_r + (lane >> 3) + 4 * k;
      if (prow >= R) continue;
      float* d = dst + (long long)prow * P.ld_final + col;
      if (col + 4 <= C) {
        *reinterpret_cast<float4*>(d) = v[k];
      } else {
        const float e[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (col + j < C) d[j] = e[j];
      }
    }
  }
}

// Waits, bounded by limit_ns, until the counter reaches `need`; acquire at
// GPU scope.
__device__ __forceinline__ bool wait_count(const int* p, int need, uint64_t limit_ns) {
  if (ld_acquire_gpu(p) >= need) return true;
  const uint64_t t0 = global_timer_ns();
  for (;;) {
    __nanosleep(64);
    if (ld_acquire_gpu(p) >= need) return true;
    if (global_timer_ns() - t0 > limit_ns) return false;
  }
}

// OPS names the operations the launch's tiles may have: one (a per-phase
// launch, or the final update: the operation is then a compile-time constant
// and the kernel carries only that epilogue) or all three (the chain launch,
// which reads each tile's operation).
constexpr int OPS_GRAM = 1 << OP_GRAM, OPS_POLY = 1 << OP_POLY, OPS_UPDATE = 1 << OP_UPDATE;
constexpr int OPS_ALL = OPS_GRAM | OPS_POLY | OPS_UPDATE;

template <int OPS>
__device__ __forceinline__ int tile_op(const NsTile& t) {
  if constexpr (OPS == OPS_GRAM) return OP_GRAM;
  else if constexpr (OPS == OPS_POLY) return OP_POLY;
  else if constexpr (OPS == OPS_UPDATE) return OP_UPDATE;
  else return t.op;
}

// Held K slices.  In the one-phase polynomial launch the epilogue input is
// a block of this CTA's own A operand: B = b A + c A^2 needs A(I, J), which
// is its A slice (rows I) for the K range J.  Those slices come last in the
// tile's K order (the order starts right after them and wraps), stay in the
// ring until the epilogue has read them, and the epilogue, not the MMA
// commit, releases them, so the input never comes from L2.  start: the
// slice at position 0; nheld: how many.
template <int OPS, bool FINAL>
__device__ __forceinline__ void hold_range(const NsTile& t, int& start, int& nheld) {
  start = 0;
  nheld = 0;
  if constexpr (!FINAL && OPS == OPS_POLY) {
    const int lo = t.j0 / BK;
    const int hi = min(lo + HOLD_CHUNKS, t.kc);
    nheld = max(hi - lo, 0);
    start = hi < t.kc ? hi : 0;
  }
}

template <int OPS, bool FINAL, bool MIRROR = false>
__device__ __forceinline__ void ns_gemm_body(const NsLaunch& L, const FinalTable* F) {
  constexpr int NST = FINAL ? (MIRROR ? FINAL_STAGES : REDUCE_STAGES)
                            : STAGES;   // ring depth
  constexpr int EPI_REGION = FINAL ? (MIRROR ? FINAL_EPI_BYTES : REDUCE_EPI_BYTES)
                                   : EPI_STAGE_BYTES;                          // per epilogue warp
  constexpr bool HOLD = !FINAL && OPS == OPS_POLY;   // see hold_range
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;     // 128B-swizzle atoms need 1 KB alignment
  uint8_t* gbase = smem_raw + (sbase - raw);
  const uint32_t bar0 = sbase + NST * STAGE_BYTES + EPI_WARPS * EPI_REGION;
  // barrier layout: full[NST], empty[NST], tfull[2], tempty[2], drain,
  // then (final kernel) P_RING parameter-block barriers per epilogue warp
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (NST + s); };
  auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * NST + a); };
  auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * NST + 2 + a); };
  const uint32_t drain_bar = bar0 + 8u * (2 * NST + 4);
  const uint32_t pbar_base = bar0 + 8u * (2 * NST + 5);
  constexpr int NBARS = 2 * NST + 5 + (FINAL ? EPI_WARPS * P_RING : 0);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + NST * STAGE_BYTES +
                                                    EPI_WARPS * EPI_REGION + 8 * NBARS);
  // Per stage: epilogue warps done reading it as a held slice (four per use).
  int* hold_cnt = reinterpret_cast<int*>(tmem_slot + 2);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // CTA pair: rank 0 (the leader) issues every MMA of the pair and owns the
  // barriers the MMA waits on; both CTAs load their own operand halves and
  // run their own epilogue on their own TMEM rows.
  const uint32_t rank = cluster_cta_rank();
  const bool leader = rank == 0;
  const int pair = (int)(blockIdx.x >> 1);
  const int npairs = (int)(gridDim.x >> 1);

  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(full_bar(s), 1);        // leader: its producer arms; both CTAs' bytes land
      mbar_init(empty_bar(s), 1);       // both: the leader's MMA commit (multicast)
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);                    // both: leader's commit (multicast)
      mbar_init(tempty_bar(a), 2 * EPI_THREADS);     // leader: both CTAs' epilogues
    }
    mbar_init(drain_bar, 1);
    if (HOLD)
      for (int s = 0; s < NST; ++s) hold_cnt[s] = 0;
    if (FINAL)
      for (int b = 0; b < EPI_WARPS * P_RING; ++b) mbar_init(pbar_base + 8u * b, 1);
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_addr(tmem_slot), TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before_sync();
  cluster_sync_all();            // both CTAs: barriers initialised, TMEM allocated
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const unsigned long long limit = L.limit_ns;

  // Checked builds: both CTAs of the pair validate every tile the pair owns
  // (the same list, so they agree) and refuse all of them if one is invalid.
  bool refuse = false;
  if (kBoundsCheck) {
    int bad = 0;
    for (int t = pair + (int)threadIdx.x * npairs; t < L.ntiles; t += (int)blockDim.x * npairs) {
      const NsTile tl = L.tiles[t];
      bool ok = tl.prob >= 0 && tl.prob < L.nprobs && tl.op >= OP_GRAM && tl.op <= OP_UPDATE &&
                (FINAL ? tl.op == OP_UPDATE : true) && tl.wait_idx < L.ndeps && tl.done_idx < L.ndeps;
      if (ok) {
        const NsProblem& Q = L.probs[tl.prob];
        ok = tl.i0 >= 0 && tl.i0 < Q.M && tl.j0 >= 0 && tl.j0 < Q.N && tl.kc > 0 &&
             (long long)tl.kc * BK >= Q.K && Q.slot >= 0 && Q.slot < MUON_MAX_GROUP;
      }
      bad |= ok ? 0 : 1;
    }
    refuse = __syncthreads_or(bad) != 0;
    if (refuse && threadIdx.x == 0) record_status(L.status, MUON_ERR_INVALID_ARG);
  }

  if (refuse) {
    // nothing issued: straight to the teardown
  } else if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer (both CTAs)
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed_mask = 0, armed_parity = 0;   // leader: stages it armed
      uint32_t used_mask = 0, used_parity = 0;     // stages this CTA loaded into
      bool ok = true;
      for (int t = pair; t < L.ntiles && ok; t += npairs) {
        const NsTile tile = L.tiles[t];
        const NsProblem* P = L.probs + tile.prob;
        if (tile.wait_idx >= 0) {
          // The operands were written by the previous phase in this launch.
          if (!wait_count(L.deps + tile.wait_idx, tile.wait_need, limit)) {
            record_status(L.status, MUON_ERR_TIMEOUT);
            ok = false;
            break;
          }
          fence_proxy_async();                     // ... and TMA must see them
        }
        const int op = tile_op<OPS>(tile);
        const int arow = tile.i0 + (int)rank * BM;           // this CTA's rows of A
        const int bcol = tile.j0 + (int)rank * (BN / 2);     // this CTA's half of B
        // A diagonal tile of a symmetric product (Gram, polynomial): both
        // operands are rows of one matrix and this CTA's half of B is its own
        // rows of A, so the B slice is not loaded; the MMA reads it from A.
        const bool same_ab = op != OP_UPDATE && tile.i0 == tile.j0;
        int kstart, nheld;
        hold_range<OPS, FINAL>(tile, kstart, nheld);
        for (int kc = 0; kc < tile.kc; ++kc) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, limit)) {
            record_status(L.status, MUON_ERR_TIMEOUT);
            ok = false;
            break;
          }
          if (leader) {
            mbar_arrive_expect_tx(full_bar(stage), same_ab ? 2 * A_STAGE_BYTES : 2 * STAGE_BYTES);
            armed_mask |= 1u << stage;
            armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
          }
          used_mask |= 1u << stage;
          used_parity = (used_parity & ~(1u << stage)) | (phase << stage);
          const uint32_t fb = map_to_cta(full_bar(stage), 0);   // the leader's barrier
          const uint32_t sA = sbase + stage * STAGE_BYTES;
          const uint32_t sB = sA + A_STAGE_BYTES;
          const int kslice = kstart + kc < tile.kc ? kstart + kc : kstart + kc - tile.kc;
          const int k0 = kslice * BK;
#pragma unroll
          for (int q = 0; q < BM / BOX; ++q)
            tma_load_2d_pair(sA + q * BOX_BYTES, &P->tmA, fb, k0, arow + q * BOX);
          if (op == OP_UPDATE) {
            // B operand = X[k0:k0+64, bcol:bcol+128], MN-major: boxes along columns.
#pragma unroll
            for (int q = 0; q < (BN / 2) / BOX; ++q)
              tma_load_2d_pair(sB + q * BOX_BYTES, &P->tmB, fb, bcol + q * BOX, k0);
          } else if (!same_ab) {
            // B operand = rows bcol..bcol+128 of X (or A), K-major.
#pragma unroll
            for (int q = 0; q < (BN / 2) / BOX; ++q)
              tma_load_2d_pair(sB + q * BOX_BYTES, &P->tmB, fb, k0, bcol + q * BOX);
          }
          if (++stage == NST) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // Never leave with copies in flight.  The leader waits for the last
      // phase it armed on each stage (both CTAs' bytes land there); the peer
      // waits for the MMA commit that follows its last load of each stage.
      // On the normal path all of these have completed already.
      for (int s = 0; s < NST; ++s) {
        if (leader && (armed_mask & (1u << s)))
          if (!mbar_wait(full_bar(s), (armed_parity >> s) & 1u, kDrainLimitNs))
            record_status(L.status, MUON_ERR_TIMEOUT);
        if (!leader && (used_mask & (1u << s)))
          if (!mbar_wait(empty_bar(s), (used_parity >> s) & 1u, kDrainLimitNs))
            record_status(L.status, MUON_ERR_TIMEOUT);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ------------------------------------------------ MMA issuer (leader only)
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int t = pair; t < L.ntiles && ok; t += npairs) {
        const NsTile tile = L.tiles[t];
        const bool mn = tile_op<OPS>(tile) == OP_UPDATE;
        const bool same_ab = !mn && tile.i0 == tile.j0;   // B slice = A slice (see producer)
        const uint32_t idesc = mn ? kIdescMN : kIdescK;
        int kstart, nheld;
        hold_range<OPS, FINAL>(tile, kstart, nheld);
        if (!mbar_wait(tempty_bar(acc), acc_phase ^ 1u, limit)) {
          record_status(L.status, MUON_ERR_TIMEOUT);
          break;
        }
        tc_fence_after_sync();
        const uint32_t d_tmem = tmem + acc * BN;
        for (int kc = 0; kc < tile.kc; ++kc) {
          if (!mbar_wait(full_bar(stage), phase, limit)) {
            record_status(L.status, MUON_ERR_TIMEOUT);
            ok = false;
            break;
          }
          tc_fence_after_sync();
          const uint32_t sA = sbase + stage * STAGE_BYTES;
          const uint32_t sB = same_ab ? sA : sA + A_STAGE_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            // K-major A: 128-byte rows, 8-row groups 1 KB apart; a K step of
            // 16 elements moves the start 32 bytes inside the swizzle atom.
            const uint64_t adesc = smem_desc_sw128(sA + kk * 32, 16, 1024);
            uint64_t bdesc;
            if (mn) {
              // MN-major B: 64-column blocks one box (8 KB) apart, 8-row K
              // groups 1 KB apart; a K step of 16 rows moves 2 KB.
              bdesc = smem_desc_sw128(sB + kk * 2048, BOX_BYTES, 1024);
            } else {
              bdesc = smem_desc_sw128(sB + kk * 32, 16, 1024);
            }
            umma_f16_pair(d_tmem, adesc, bdesc, idesc, (kc | kk) != 0 ? 1u : 0u);
          }
          if (kc < tile.kc - nheld) umma_commit_pair(empty_bar(stage), 0x3);   // both CTAs' slices free
          if (++stage == NST) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit_pair(tfull_bar(acc), 0x3);       // both CTAs' accumulators ready
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      // Drain: every MMA issued above completes before TMEM is released.
      umma_commit_pair(drain_bar, 0x1);
      if (!mbar_wait(drain_bar, 0, kDrainLimitNs)) record_status(L.status, MUON_ERR_TIMEOUT);
    }
  } else {
    // -------------------------------------------------- epilogue (warps 2-9)
    const int ew = warp - 2;                    // 0..7
    const int quarter = warp & 3;               // TMEM lanes this warp may access
    const int half = ew >> 2;                   // which 4 of the 8 column chunks
    uint8_t* stg8 = gbase + NST * STAGE_BYTES + ew * EPI_REGION;
    uint16_t* stg = reinterpret_cast<uint16_t*>(stg8);
    const uint32_t stg_s = smem_addr(stg8);
    if (FINAL && L.pmaps != nullptr && L.final_mode == FINAL_PARAM) {
      // ---- last iteration, the parameter update through the TMA.
      // Without mirrors the epilogue never reads the parameters: it writes
      // the increment d = fp32(-lr s X) of each 32 x 32 block into a
      // shared-memory block and a TMA reduce-add makes the memory system add
      // it to p (p <- fp32(p + d)).  Chunk h uses block h % 2, last used by
      // chunk h - 2, whose reduce has finished reading it once at most one
      // bulk group (chunk h - 1's) still reads.
      // With mirrors the final values are needed here, so the parameter
      // blocks come through a per-warp ring of TMA loads: chunk h owns ring
      // slot h % P_RING; the block for chunk h + P_AHEAD is loaded while
      // chunk h is combined; that slot last held chunk h + P_AHEAD - P_RING =
      // h - 2, whose store has finished reading once at most one store group
      // (chunk h - 1's) is still reading.  Both forms compute fp32(p + d).
      uint8_t* ring = stg8;
      const uint32_t ring_s = smem_addr(ring);
      const uint32_t pbar0 = pbar_base + 8u * (ew * P_RING);
      const int ntl = (pair < L.ntiles) ? (L.ntiles - 1 - pair) / npairs + 1 : 0;
      const int nch = ntl * CHUNKS_PER_WARP;
      uint32_t pphase = 0;    // per slot: parity of its next completion
      uint32_t pending = 0;   // per slot: a load is in flight and not yet consumed
      auto chunk_info = [&](int h, const NsProblem*& Pp, int& rb, int& c0) -> bool {
        const NsTile tl = L.tiles[pair + (h / CHUNKS_PER_WARP) * npairs];
        Pp = L.probs + tl.prob;
        rb = tl.i0 + (int)rank * BM + quarter * 32;
        c0 = tl.j0 + half * (CHUNKS_PER_WARP * 32) + (h % CHUNKS_PER_WARP) * 32;
        return rb < Pp->M && c0 < Pp->N;
      };
      auto issue = [&](int h) {          // every lane tracks the state; lane 0 issues
        if (!MIRROR || h >= nch) return;
        const NsProblem* Pp;
        int rb, c0;
        if (!chunk_info(h, Pp, rb, c0)) return;
        const int b = h % P_RING;
        if (lane == 0) {
          const uint32_t bar = pbar0 + 8u * b;
          mbar_arrive_expect_tx(bar, P_BLOCK_BYTES);
          const CUtensorMap* pm = L.pmaps + Pp->slot;
          // transposed targets: X(i, j) is p[j][i], so the block starts at p(col0, rbase)
          if (Pp->transposed) tma_load_2d(ring_s + b * P_BLOCK_BYTES, pm, bar, rb, c0);
          else tma_load_2d(ring_s + b * P_BLOCK_BYTES, pm, bar, c0, rb);
        }
        pending |= 1u << b;
      };
      for (int h = 0; h < P_AHEAD; ++h) issue(h);
      // The epilogue input (a X) of chunk h + E_AHEAD is loaded while chunk
      // h is combined, across tile boundaries, from a ring of registers:
      // eb[0] is the current chunk's.
      uint4 eb[E_AHEAD + 1][4];
      auto in_load = [&](int h, uint4 (&dst)[4]) {
        if (h >= nch) return;
        const NsProblem* Pp;
        int rb, c0;
        chunk_info(h, Pp, rb, c0);
        load_row(Pp->epi, Pp->ld_epi, rb + lane, c0, Pp->M, Pp->N, dst);
      };
#pragma unroll
      for (int k = 0; k < E_AHEAD; ++k) in_load(k, eb[k]);
      int acc = 0;
      uint32_t acc_phase = 0;
      for (int h = 0; h < nch; ++h) {
        const int cc = h % CHUNKS_PER_WARP;
        const NsProblem* Pp;
        int rb, col0;
        const bool live = chunk_info(h, Pp, rb, col0);
        const NsProblem& P = *Pp;
        if (cc == 0) {
          if (!mbar_wait(tfull_bar(acc), acc_phase, limit)) {
            record_status(L.status, MUON_ERR_TIMEOUT);
            break;
          }
          tc_fence_after_sync();
        }
        if (lane == 0) bulk_wait_group_read<1>();   // the store of chunk h - 2 has read its slot
        __syncwarp();
        issue(h + P_AHEAD);
        in_load(h + E_AHEAD, eb[E_AHEAD]);
        uint32_t v[32];
        tmem_ld_32x32b_x32(tmem + (static_cast<uint32_t>(quarter * 32) << 16) + acc * BN +
                               half * (CHUNKS_PER_WARP * 32) + cc * 32, v);
        tmem_ld_wait();
        bool stop = false;
        if (live) {
          const int b = MIRROR ? h % P_RING : (h & 1);
          bool got = true;
          if (MIRROR) {
            got = mbar_wait(pbar0 + 8u * b, (pphase >> b) & 1u, limit);
            pphase ^= 1u << b;
            pending &= ~(1u << b);
          }
          if (!got) {
            record_status(L.status, MUON_ERR_TIMEOUT);
            stop = true;
          } else {
            float in[32], xb[32];
#pragma unroll
            for (int q = 0; q < 4; ++q) unpack8(eb[0][q], in + 8 * q);
#pragma unroll
            for (int c = 0; c < 32; ++c)
              xb[c] = __bfloat162float(__float2bfloat16_rn(fmaf(L.ca, in[c], __uint_as_float(v[c]))));
            const float neg_scale = -F->scale[P.slot];
            uint8_t* blk = ring + b * P_BLOCK_BYTES;
            // 32 x 32 fp32 block, 128-byte swizzle: element (r, c) at
            // r*128 + (((c >> 2) ^ (r & 7)) << 4) + (c & 3)*4
            if (P.transposed) {
              // this lane's X row is block column `lane`; X column c is block row c
#pragma unroll
              for (int c = 0; c < 32; ++c) {
                float* q = reinterpret_cast<float*>(blk + c * 128 + ((((lane >> 2) ^ (c & 7))) << 4) +
                                                    ((lane & 3) << 2));
                const float d = __fmul_rn(neg_scale, xb[c]);
                *q = MIRROR ? __fadd_rn(*q, d) : d;
              }
            } else {
#pragma unroll
              for (int qd = 0; qd < 8; ++qd) {
                float4* q = reinterpret_cast<float4*>(blk + lane * 128 + ((qd ^ (lane & 7)) << 4));
                float4 d = make_float4(__fmul_rn(neg_scale, xb[4 * qd + 0]),
                                       __fmul_rn(neg_scale, xb[4 * qd + 1]),
                                       __fmul_rn(neg_scale, xb[4 * qd + 2]),
                                       __fmul_rn(neg_scale, xb[4 * qd + 3]));
                if (MIRROR) {
                  const float4 pv = *q;
                  d = make_float4(__fadd_rn(pv.x, d.x), __fadd_rn(pv.y, d.y), __fadd_rn(pv.z, d.z),
                                  __fadd_rn(pv.w, d.w));
                }
                *q = d;
              }
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              const CUtensorMap* pm = L.pmaps + P.slot;
              const uint32_t src = ring_s + b * P_BLOCK_BYTES;
              if (MIRROR) {
                if (P.transposed) tma_store_2d(pm, src, rb, col0);
                else tma_store_2d(pm, src, col0, rb);
              } else {
                if (P.transposed) tma_reduce_add_2d(pm, src, rb, col0);
                else tma_reduce_add_2d(pm, src, col0, rb);
              }
            }
            if constexpr (MIRROR) {
              // The block is final in shared memory (only read from here on,
              // by this warp and the TMA store), so the lanes copy it out too.
              if (P.transposed) mirror_block(L, P, blk, col0, rb, lane);
              else mirror_block(L, P, blk, rb, col0, lane);
            }
          }
        }
        if (lane == 0) bulk_commit_group();        // one group per chunk, empty or not
        if (stop) break;
#pragma unroll
        for (int k = 0; k < E_AHEAD; ++k)
#pragma unroll
          for (int q = 0; q < 4; ++q) eb[k][q] = eb[k + 1][q];
        if (cc + 1 == CHUNKS_PER_WARP) {
          tc_fence_before_sync();
          mbar_arrive_remote(map_to_cta(tempty_bar(acc), 0));
          if (++acc == 2) {
            acc = 0;
            acc_phase ^= 1u;
          }
        }
      }
      // Loads issued but never consumed (only after a timeout) land before exit.
      for (int b = 0; b < P_RING; ++b)
        if (pending & (1u << b))
          if (!mbar_wait(pbar0 + 8u * b, (pphase >> b) & 1u, kDrainLimitNs))
            record_status(L.status, MUON_ERR_TIMEOUT);
    } else {
    int acc = 0;
    uint32_t acc_phase = 0;
    int it = 0;     // ring position of the tile's first K slice (as producer and MMA count)
    for (int t = pair; t < L.ntiles; t += npairs) {
      const NsTile tile = L.tiles[t];
      const NsProblem& P = L.probs[tile.prob];
      const int op = tile_op<OPS>(tile);
      const int M = P.M, N = P.N;
      int kstart, nheld;
      hold_range<OPS, FINAL>(tile, kstart, nheld);
      const int held0 = it + tile.kc - nheld;      // ring position of the first held slice
      it += tile.kc;
      const int rbase = tile.i0 + (int)rank * BM + quarter * 32;
      const int row = rbase + lane;
      const int cbase = tile.j0 + half * (CHUNKS_PER_WARP * 32);
      // Epilogue input (this lane's row), fetched before the accumulator is
      // ready; in a chain launch only once the phase that wrote it is done.
      // The lanes wait independently (lane 0 may still be counting the last
      // tile) and agree on failure in one vote before any warp-wide step.
      bool fail = !FINAL && op != OP_GRAM && tile.wait_idx >= 0 &&
                  !wait_count(L.deps + tile.wait_idx, tile.wait_need, limit);
      const int npre = fail ? 0 : (op == OP_GRAM || HOLD) ? 0 : (FINAL ? 1 : CHUNKS_PER_WARP);
      uint4 ein[FINAL ? 1 : CHUNKS_PER_WARP][4];
#pragma unroll
      for (int cc = 0; cc < (FINAL ? 1 : CHUNKS_PER_WARP); ++cc)
        if (cc < npre) load_row<OPS == OPS_ALL>(P.epi, P.ld_epi, row, cbase + cc * 32, M, N, ein[cc]);
      float pcur[32];
      if (FINAL) final_load(P, F, L.final_mode, rbase, cbase, lane, pcur);
      if (!fail) fail = !mbar_wait(tfull_bar(acc), acc_phase, limit);
      if (__any_sync(0xffffffffu, fail)) {
        record_status(L.status, MUON_ERR_TIMEOUT);
        break;
      }
      tc_fence_after_sync();
      if (HOLD) {
        // Every MMA of the tile has completed: the held slices are read here
        // (this half's two) and released, the fourth reader warp of a slice
        // arriving on its empty barrier.
#pragma unroll
        for (int cc = 0; cc < CHUNKS_PER_WARP; ++cc) {
          const int ci = half * (CHUNKS_PER_WARP / 2) + (cc >> 1);
          if (ci < nheld) {
            held_row(gbase + ((held0 + ci) % NST) * STAGE_BYTES, quarter * 32 + lane, (cc & 1) * 32,
                     ein[cc]);
          }
        }
        __syncwarp();
        if (lane == 0) {
#pragma unroll
          for (int u = 0; u < CHUNKS_PER_WARP / 2; ++u) {
            const int ci = half * (CHUNKS_PER_WARP / 2) + u;
            if (ci < nheld) {
              const int s = (held0 + ci) % NST;
              __threadfence_block();
              if ((atomicAdd(hold_cnt + s, 1) & 3) == 3) {
                __threadfence_block();
                mbar_arrive(empty_bar(s));
              }
            }
          }
        }
      }
      const uint32_t tbase = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + acc * BN +
                             half * (CHUNKS_PER_WARP * 32);
      const bool rows_live = rbase < M;
      if (FINAL) {
        // Last iteration: one chunk of input and parameters in flight ahead.
#pragma unroll 1
        for (int cc = 0; cc < CHUNKS_PER_WARP; ++cc) {
          const int col0 = cbase + cc * 32;
          uint4 enext[4];
          float pnext[32];
          if (cc + 1 < CHUNKS_PER_WARP) {
            load_row(P.epi, P.ld_epi, row, col0 + 32, M, N, enext);
            final_load(P, F, L.final_mode, rbase, col0 + 32, lane, pnext);
          }
          uint32_t v[32];
          tmem_ld_32x32b_x32(tbase + cc * 32, v);
          tmem_ld_wait();
          if (rows_live && col0 < N) {                // warp-uniform
            float in[32], xb[32];
#pragma unroll
            for (int q = 0; q < 4; ++q) unpack8(ein[0][q], in + 8 * q);
#pragma unroll
            for (int c = 0; c < 32; ++c)
              xb[c] = __bfloat162float(__float2bfloat16_rn(fmaf(L.ca, in[c], __uint_as_float(v[c]))));
            final_apply(P, F, L.final_mode, stg, xb, rbase, col0, lane, pcur);
          }
          if (cc + 1 < CHUNKS_PER_WARP) {
#pragma unroll
            for (int q = 0; q < 4; ++q) ein[0][q] = enext[q];
#pragma unroll
            for (int c = 0; c < 32; ++c) pcur[c] = pnext[c];
          }
        }
      } else {
#pragma unroll
      for (int cc = 0; cc < CHUNKS_PER_WARP; ++cc) {
        const int col0 = cbase + cc * 32;
        uint4 (&ecur)[4] = ein[FINAL ? 0 : cc];
        uint32_t v[32];
        tmem_ld_32x32b_x32(tbase + cc * 32, v);
        tmem_ld_wait();
        if (!rows_live || col0 >= N) continue;     // warp-uniform
        float x[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) x[c] = __uint_as_float(v[c]);
        if (op != OP_GRAM) {
          float in[32];
#pragma unroll
          for (int q = 0; q < 4; ++q) unpack8(ecur[q], in + 8 * q);
          if (op == OP_POLY) {
#pragma unroll
            for (int c = 0; c < 32; ++c) x[c] = fmaf(L.cc, x[c], L.cb * in[c]);
          } else {
#pragma unroll
            for (int c = 0; c < 32; ++c) x[c] = fmaf(L.ca, in[c], x[c]);
          }
        }
        if (op == OP_GRAM || op == OP_POLY) {
          // Symmetric output.  rbase and col0 are multiples of 32, so this
          // block lies above the diagonal (stored and mirrored), on it
          // (symmetrised, stored once) or below it (owned by another tile).
          if (col0 < rbase) continue;
          if (lane == 0) bulk_wait_group_read<0>();    // both blocks free again
          __syncwarp();
          row_to_block(stg8, lane, x);
          if (col0 == rbase) {
            __syncwarp();
            symmetrize_block(stg8, lane);
          } else {
            col_to_block(stg8 + EPI_BLOCK_BYTES, lane, x);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&P.tmOut, stg_s, col0, rbase);
            if (col0 != rbase) tma_store_2d(&P.tmOut, stg_s + EPI_BLOCK_BYTES, rbase, col0);
            bulk_commit_group();
          }
        } else {
          // X update: two chunks fill one 32 x 64 block, which leaves in one
          // TMA store (half as many stores as 32 x 32 blocks).
          if ((cc & 1) == 0) {
            if (lane == 0) bulk_wait_group_read<0>();  // the last block's store has read it
            __syncwarp();
          }
          row_to_wide(stg8, lane, cc & 1, x);
          if ((cc & 1) == 1 || cc + 1 == CHUNKS_PER_WARP || col0 + 32 >= N) {
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_2d(&P.tmOut, stg_s, col0 - (cc & 1) * 32, rbase);
              bulk_commit_group();
            }
          }
        }
      }
      }
      tc_fence_before_sync();
      mbar_arrive_remote(map_to_cta(tempty_bar(acc), 0));   // the leader's MMA waits on it
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
      if (!FINAL && tile.done_idx >= 0 && lane == 0) {
        // Once this warp's stores of the tile have landed, count them for
        // the next phase (each of the pair's 16 epilogue warps once per
        // tile).  Only lane 0 waits; the other lanes go on to the next
        // tile's input and accumulator, where lane 0 catches up.
        bulk_wait_group_all();
        fence_proxy_async();
        red_release_gpu_add(L.deps + tile.done_idx, 1);
      }
    }
    }
    // Stores must finish reading shared memory (and land) before the CTA exits.
    if (lane == 0) bulk_wait_group_all();
    if constexpr (MIRROR) __threadfence_system();   // mirror stores, possibly to peers
    __syncwarp();
  }

  // Both CTAs finished: no MMA writes either TMEM and no arrival targets
  // either CTA's barriers any more.
  tc_fence_before_sync();
  cluster_sync_all();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after_sync();
    tmem_dealloc_pair(tmem, TMEM_COLS);
  }
}

// Gram, polynomial or X-update tiles: one phase per launch (OPS one
// operation), or the whole chain of phases (OPS_ALL).
template <int OPS>
__global__ void __launch_bounds__(GEMM_THREADS, 1) ns_gemm_kernel(const __grid_constant__ NsLaunch L) {
  ns_gemm_body<OPS, false>(L, nullptr);
}

__global__ void __launch_bounds__(GEMM_THREADS, 1)
    ns_gemm_final_kernel(const __grid_constant__ NsLaunch L, const __grid_constant__ FinalTable F) {
  ns_gemm_body<OPS_UPDATE, true>(L, &F);
}

// The last update that also writes every parameter block to its mirrors.
__global__ void __launch_bounds__(GEMM_THREADS, 1)
    ns_gemm_final_mirror_kernel(const __grid_constant__ NsLaunch L,
                                const __grid_constant__ FinalTable F) {
  ns_gemm_body<OPS_UPDATE, true, true>(L, &F);
}

}  // namespace

cudaError_t ns_gemm_setup(int /*device*/) {
  cudaError_t e;
  for (auto k : {ns_gemm_kernel<OPS_GRAM>, ns_gemm_kernel<OPS_POLY>, ns_gemm_kernel<OPS_UPDATE>,
                 ns_gemm_kernel<OPS_ALL>}) {
    e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)GEMM_SMEM_BYTES);
    if (e != cudaSuccess) return e;
  }
  e = cudaFuncSetAttribute(ns_gemm_final_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)REDUCE_SMEM_BYTES);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(ns_gemm_final_mirror_kernel,
                              cudaFuncAttributeMaxDynamicSharedMemorySize, (int)FINAL_SMEM_BYTES);
}

// How many CTA pairs (clusters of two) can be resident at once.
int ns_gemm_max_pairs() {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2);
  cfg.blockDim = dim3(GEMM_THREADS);
  cfg.dynamicSmemBytes = GEMM_SMEM_BYTES;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, ns_gemm_kernel<OPS_ALL>, &cfg) != cudaSuccess || n < 1) {
    cudaGetLastError();
    return 0;
  }
  return n;
}

// Launched as clusters of two CTAs (the MMA pair); grid is even.  `op` is
// the one operation of every tile, or -1 for a chain launch (tiles of all
// three, waiting on one another), which is cooperative so that every CTA a
// wait depends on is resident at the same time.
cudaError_t launch_ns_gemm(const NsLaunch& L, const FinalTable* F, int grid, cudaStream_t stream,
                           int op) {
  const bool cooperative = op < 0;
  if (L.ntiles <= 0) return cudaSuccess;
  const bool fin = L.final_mode != FINAL_NONE;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(GEMM_THREADS);
  cfg.dynamicSmemBytes = fin ? (L.n_mirrors > 0 ? FINAL_SMEM_BYTES : REDUCE_SMEM_BYTES)
                             : GEMM_SMEM_BYTES;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeCooperative;
  attr[1].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = cooperative ? 2 : 1;
  if (!fin) {
    if (op == OP_GRAM) return cudaLaunchKernelEx(&cfg, ns_gemm_kernel<OPS_GRAM>, L);
    if (op == OP_POLY) return cudaLaunchKernelEx(&cfg, ns_gemm_kernel<OPS_POLY>, L);
    if (op == OP_UPDATE) return cudaLaunchKernelEx(&cfg, ns_gemm_kernel<OPS_UPDATE>, L);
    return cudaLaunchKernelEx(&cfg, ns_gemm_kernel<OPS_ALL>, L);
  }
  if (L.n_mirrors > 0) {
    // Mirrors are written only from the shared-memory parameter ring.
    if (L.final_mode != FINAL_PARAM || L.pmaps == nullptr) return cudaErrorInvalidValue;
    return cudaLaunchKernelEx(&cfg, ns_gemm_final_mirror_kernel, L, *F);
  }
  return cudaLaunchKernelEx(&cfg, ns_gemm_final_kernel, L, *F);
}

}  // namespace muon
