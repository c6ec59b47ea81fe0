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
// matrix of the phase as one grouped launch.  Per CTA:
//   warp 0     one thread issues TMA tile loads (64x64 bf16 boxes, 128-byte
//              swizzle) into a STAGES-deep ring of shared-memory slices;
//   warp 1     one thread issues tcgen05.mma (M=128, N=256, K=16, fp32
//              accumulation in TMEM) and commits slices back to the ring;
//   warps 2-5  read the accumulator from TMEM (tcgen05.ld), apply the fp32
//              epilogue and store bf16 (or the fp32 parameter update).
// Two TMEM accumulators (2 x 256 columns) let the epilogue of one tile
// overlap the main loop of the next.  Every wait is bounded.
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

constexpr uint32_t kIdescK = idesc_bf16_f32(BM, BN, 0);   // B operand K-major
constexpr uint32_t kIdescMN = idesc_bf16_f32(BM, BN, 1);  // B operand MN-major

__device__ __forceinline__ void record_status(int* status, int code) {
  atomicCAS(status, 0, code);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Loads 32 bf16 values at row `row`, columns [col0, col0+32) of a row-major
// matrix (leading dimension ld) as floats; columns >= N read as 0.
__device__ __forceinline__ void load_row32(const __nv_bfloat16* base, long long ld, int row,
                                           int col0, int N, float (&o)[32]) {
  const __nv_bfloat16* p = base + (long long)row * ld + col0;
  if (col0 + 32 <= N) {
    const uint4* q = reinterpret_cast<const uint4*>(p);
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      uint4 w = __ldg(q + v);
      uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        o[v * 8 + 2 * t] = bf16_bits_to_float(u[t] & 0xFFFFu);
        o[v * 8 + 2 * t + 1] = bf16_bits_to_float(u[t] >> 16);
      }
    }
  } else {
#pragma unroll
    for (int c = 0; c < 32; ++c)
      o[c] = (col0 + c < N) ? __bfloat162float(p[c]) : 0.f;
  }
}

template <int OP>
__device__ __forceinline__ void epilogue_chunk(const NsLaunch& L, const NsProblem& P,
                                               const FinalTable* F, int row, int col0,
                                               const uint32_t (&acc)[32]) {
  const int M = P.M, N = P.N;
  if (row >= M || col0 >= N) return;
  float x[32];
#pragma unroll
  for (int c = 0; c < 32; ++c) x[c] = __uint_as_float(acc[c]);

  if (OP == OP_POLY) {
    float a[32];
    load_row32(P.epi, P.ld_epi, row, col0, N, a);
#pragma unroll
    for (int c = 0; c < 32; ++c) x[c] = fmaf(L.cc, x[c], L.cb * a[c]);
  } else if (OP == OP_UPDATE) {
    float a[32];
    load_row32(P.epi, P.ld_epi, row, col0, N, a);
#pragma unroll
    for (int c = 0; c < 32; ++c) x[c] = fmaf(L.ca, a[c], x[c]);
  }

  if (OP == OP_GRAM || OP == OP_POLY) {
    // Symmetric output: entry (row, col) is owned by the tile computing it
    // with col >= row; it is stored there and mirrored to (col, row).
    __nv_bfloat16* out = P.out;
    const long long ld = P.ld_out;
    if (col0 >= row && col0 + 32 <= N) {
      uint4* q = reinterpret_cast<uint4*>(out + (long long)row * ld + col0);
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        uint4 w;
        w.x = pack_bf16x2(x[v * 8 + 0], x[v * 8 + 1]);
        w.y = pack_bf16x2(x[v * 8 + 2], x[v * 8 + 3]);
        w.z = pack_bf16x2(x[v * 8 + 4], x[v * 8 + 5]);
        w.w = pack_bf16x2(x[v * 8 + 6], x[v * 8 + 7]);
        q[v] = w;
      }
    } else {
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        const int col = col0 + c;
        if (col >= row && col < N) out[(long long)row * ld + col] = __float2bfloat16_rn(x[c]);
      }
    }
    // Mirror: lanes hold consecutive rows, so each column's 32 stores are
    // one contiguous 64-byte segment of row `col`.
#pragma unroll
    for (int c = 0; c < 32; ++c) {
      const int col = col0 + c;
      if (col > row && col < N) out[(long long)col * ld + row] = __float2bfloat16_rn(x[c]);
    }
    return;
  }

  // OP_UPDATE
  if (L.final_mode == FINAL_NONE) {
    __nv_bfloat16* out = P.out;
    const long long ld = P.ld_out;
    if (col0 + 32 <= N) {
      uint4* q = reinterpret_cast<uint4*>(out + (long long)row * ld + col0);
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        uint4 w;
        w.x = pack_bf16x2(x[v * 8 + 0], x[v * 8 + 1]);
        w.y = pack_bf16x2(x[v * 8 + 2], x[v * 8 + 3]);
        w.z = pack_bf16x2(x[v * 8 + 4], x[v * 8 + 5]);
        w.w = pack_bf16x2(x[v * 8 + 6], x[v * 8 + 7]);
        q[v] = w;
      }
    } else {
      for (int c = 0; c < 32; ++c)
        if (col0 + c < N) out[(long long)row * ld + col0 + c] = __float2bfloat16_rn(x[c]);
    }
    return;
  }

  // Final iteration: round X to bf16 (its storage precision), then write it
  // to the caller's buffer in the stored orientation or apply the update.
  float xb[32];
#pragma unroll
  for (int c = 0; c < 32; ++c) xb[c] = __bfloat162float(__float2bfloat16_rn(x[c]));
  const int slot = P.slot;
  const long long ldf = P.ld_final;
  const int mode = L.final_mode;
  const float neg_scale = -F->scale[slot];
  if (!P.transposed) {
    if (mode == FINAL_OUT_BF16) {
      __nv_bfloat16* o = reinterpret_cast<__nv_bfloat16*>(F->ptr[slot]) + (long long)row * ldf;
      for (int c = 0; c < 32; ++c)
        if (col0 + c < N) o[col0 + c] = __float2bfloat16_rn(xb[c]);
      return;
    }
    float* o = reinterpret_cast<float*>(F->ptr[slot]) + (long long)row * ldf + col0;
    const bool vec = (col0 + 32 <= N) && ((ldf & 3) == 0);
    if (mode == FINAL_PARAM) {
      if (vec) {
        float4* q = reinterpret_cast<float4*>(o);
#pragma unroll
        for (int v = 0; v < 8; ++v) {
          float4 p = q[v];
          p.x = fmaf(neg_scale, xb[4 * v + 0], p.x);
          p.y = fmaf(neg_scale, xb[4 * v + 1], p.y);
          p.z = fmaf(neg_scale, xb[4 * v + 2], p.z);
          p.w = fmaf(neg_scale, xb[4 * v + 3], p.w);
          q[v] = p;
        }
      } else {
        for (int c = 0; c < 32; ++c)
          if (col0 + c < N) o[c] = fmaf(neg_scale, xb[c], o[c]);
      }
    } else {  // FINAL_OUT_F32
      if (vec) {
        float4* q = reinterpret_cast<float4*>(o);
#pragma unroll
        for (int v = 0; v < 8; ++v)
          q[v] = make_float4(xb[4 * v], xb[4 * v + 1], xb[4 * v + 2], xb[4 * v + 3]);
      } else {
        for (int c = 0; c < 32; ++c)
          if (col0 + c < N) o[c] = xb[c];
      }
    }
    return;
  }
  // Transposed target: element (row, col) lands at [col][row]; lanes hold
  // consecutive rows, so every column is one coalesced 128-byte segment.
#pragma unroll 4
  for (int c = 0; c < 32; ++c) {
    const int col = col0 + c;
    if (col >= N) break;
    const long long off = (long long)col * ldf + row;
    if (mode == FINAL_PARAM) {
      float* o = reinterpret_cast<float*>(F->ptr[slot]) + off;
      *o = fmaf(neg_scale, xb[c], *o);
    } else if (mode == FINAL_OUT_F32) {
      reinterpret_cast<float*>(F->ptr[slot])[off] = xb[c];
    } else {
      reinterpret_cast<__nv_bfloat16*>(F->ptr[slot])[off] = __float2bfloat16_rn(xb[c]);
    }
  }
}

template <int OP>
__device__ __forceinline__ void ns_gemm_body(const NsLaunch& L, const FinalTable* F) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_addr(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;     // 128B-swizzle atoms need 1 KB alignment
  uint8_t* gbase = smem_raw + (sbase - raw);
  const uint32_t bar0 = sbase + STAGES * STAGE_BYTES;
  // barrier layout: full[STAGES], empty[STAGES], tfull[2], tempty[2], drain
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + a); };
  auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + 2 + a); };
  const uint32_t drain_bar = bar0 + 8u * (2 * STAGES + 4);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + STAGES * STAGE_BYTES + 8 * (2 * STAGES + 5));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), EPI_THREADS);
    }
    mbar_init(drain_bar, 1);
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    tmem_alloc(smem_addr(tmem_slot), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const unsigned long long limit = L.limit_ns;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed_mask = 0, armed_parity = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < L.ntiles && ok; t += gridDim.x) {
        const NsTile tile = L.tiles[t];
        const NsProblem* P = L.probs + tile.prob;
        for (int kc = 0; kc < tile.kc; ++kc) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, limit)) {
            record_status(L.status, MUON_ERR_TIMEOUT);
            ok = false;
            break;
          }
          const uint32_t fb = full_bar(stage);
          mbar_arrive_expect_tx(fb, STAGE_BYTES);
          armed_mask |= 1u << stage;
          armed_parity = (armed_parity & ~(1u << stage)) | (phase << stage);
          const uint32_t sA = sbase + stage * STAGE_BYTES;
          const uint32_t sB = sA + A_STAGE_BYTES;
          const int k0 = kc * BK;
#pragma unroll
          for (int q = 0; q < BM / BOX; ++q)
            tma_load_2d(sA + q * BOX_BYTES, &P->tmA, fb, k0, tile.i0 + q * BOX);
          if (OP == OP_UPDATE) {
            // B operand = X[k0:k0+64, j0:j0+256], MN-major: boxes along columns.
#pragma unroll
            for (int q = 0; q < BN / BOX; ++q)
              tma_load_2d(sB + q * BOX_BYTES, &P->tmB, fb, tile.j0 + q * BOX, k0);
          } else {
            // B operand = rows j0..j0+256 of X (or A), K-major.
#pragma unroll
            for (int q = 0; q < BN / BOX; ++q)
              tma_load_2d(sB + q * BOX_BYTES, &P->tmB, fb, k0, tile.j0 + q * BOX);
          }
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // Never leave with copies in flight: wait (bounded) for the last load
      // armed on each stage.  On the normal path these have all landed.
      for (int s = 0; s < STAGES; ++s)
        if (armed_mask & (1u << s))
          if (!mbar_wait(full_bar(s), (armed_parity >> s) & 1u, kDrainLimitNs))
            record_status(L.status, MUON_ERR_TIMEOUT);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------ MMA issuer
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      const uint32_t idesc = (OP == OP_UPDATE) ? kIdescMN : kIdescK;
      for (int t = blockIdx.x; t < L.ntiles && ok; t += gridDim.x) {
        const NsTile tile = L.tiles[t];
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
          const uint32_t sB = sA + A_STAGE_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            // K-major A: 128-byte rows, 8-row groups 1 KB apart; a K step of
            // 16 elements moves the start 32 bytes inside the swizzle atom.
            const uint64_t adesc = smem_desc_sw128(sA + kk * 32, 16, 1024);
            uint64_t bdesc;
            if (OP == OP_UPDATE) {
              // MN-major B: 64-column blocks one box (8 KB) apart, 8-row K
              // groups 1 KB apart; a K step of 16 rows moves 2 KB.
              bdesc = smem_desc_sw128(sB + kk * 2048, BOX_BYTES, 1024);
            } else {
              bdesc = smem_desc_sw128(sB + kk * 32, 16, 1024);
            }
            umma_f16(d_tmem, adesc, bdesc, idesc, (kc | kk) != 0 ? 1u : 0u);
          }
          umma_commit(empty_bar(stage));
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(tfull_bar(acc));
        if (++acc == 2) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      // Drain: every MMA issued above completes before TMEM is released.
      umma_commit(drain_bar);
      if (!mbar_wait(drain_bar, 0, kDrainLimitNs)) record_status(L.status, MUON_ERR_TIMEOUT);
    }
  } else {
    // -------------------------------------------------- epilogue (warps 2-5)
    const int quarter = warp & 3;               // TMEM lanes this warp may access
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = blockIdx.x; t < L.ntiles; t += gridDim.x) {
      const NsTile tile = L.tiles[t];
      const NsProblem& P = L.probs[tile.prob];
      if (!mbar_wait(tfull_bar(acc), acc_phase, limit)) {
        record_status(L.status, MUON_ERR_TIMEOUT);
        break;
      }
      tc_fence_after_sync();
      const int row = tile.i0 + quarter * 32 + lane;
      const uint32_t tbase = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + acc * BN;
#pragma unroll 1
      for (int ch = 0; ch < BN / 32; ++ch) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(tbase + ch * 32, v);
        tmem_ld_wait();
        epilogue_chunk<OP>(L, P, F, row, tile.j0 + ch * 32, v);
      }
      tc_fence_before_sync();
      mbar_arrive(tempty_bar(acc));
      if (++acc == 2) {
        acc = 0;
        acc_phase ^= 1u;
      }
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after_sync();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

template <int OP>
__global__ void __launch_bounds__(GEMM_THREADS, 1) ns_gemm_kernel(const __grid_constant__ NsLaunch L) {
  ns_gemm_body<OP>(L, nullptr);
}

__global__ void __launch_bounds__(GEMM_THREADS, 1)
    ns_gemm_final_kernel(const __grid_constant__ NsLaunch L, const __grid_constant__ FinalTable F) {
  ns_gemm_body<OP_UPDATE>(L, &F);
}

}  // namespace

cudaError_t ns_gemm_setup(int /*device*/) {
  cudaError_t e;
  e = cudaFuncSetAttribute(ns_gemm_kernel<OP_GRAM>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)GEMM_SMEM_BYTES);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(ns_gemm_kernel<OP_POLY>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)GEMM_SMEM_BYTES);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(ns_gemm_kernel<OP_UPDATE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)GEMM_SMEM_BYTES);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(ns_gemm_final_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)GEMM_SMEM_BYTES);
}

cudaError_t launch_ns_gemm(int op, const NsLaunch& L, const FinalTable* F, int grid,
                           cudaStream_t stream) {
  if (L.ntiles <= 0) return cudaSuccess;
  const dim3 g(grid), b(GEMM_THREADS);
  if (op == OP_GRAM) {
    ns_gemm_kernel<OP_GRAM><<<g, b, GEMM_SMEM_BYTES, stream>>>(L);
  } else if (op == OP_POLY) {
    ns_gemm_kernel<OP_POLY><<<g, b, GEMM_SMEM_BYTES, stream>>>(L);
  } else if (L.final_mode == FINAL_NONE) {
    ns_gemm_kernel<OP_UPDATE><<<g, b, GEMM_SMEM_BYTES, stream>>>(L);
  } else {
    ns_gemm_final_kernel<<<g, b, GEMM_SMEM_BYTES, stream>>>(L, *F);
  }
  return cudaGetLastError();
}

}  // namespace muon
