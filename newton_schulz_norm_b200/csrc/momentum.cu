// momentum.cu -- the HBM-bound first kernel of the Muon step, and the
// elementwise update used when no Newton-Schulz iteration runs.
//
// Per matrix (stored r x c, fp32):
//   buf <- beta*buf + g                 ("07. Training neural networks",
//                                        section "Momentum": PyTorch form)
//   u    = g + beta*buf  (Nesterov)     (X thread, tweet 5/8: orthogonalise
//   u    = buf           (plain)         the update after Nesterov momentum)
//   nu   = ||u||_F
//   X0   = bf16(u / (nu + 1e-7)), stored transposed when r > c.
//
// The norm needs the whole matrix before any element can be cast, so the
// kernel works in two passes over 64 x 64 tiles, fed by one work queue of
// items (four tiles each):
//   pass 1 (item): momentum, write buf, partial sum of squares;
//   pass 2 (item): wait until the matrix's norm is published, recompute u
//                  from g and the new buf, scale, cast, (transpose,) store.
// The host queues a matrix's pass-2 items about half a wave of CTAs after its
// last pass-1 item, behind pass-1 items of later matrices: late enough that
// the norm is usually published when they are reached, early enough that
// pass 2 re-reads g and buf mostly from L2.  The last pass-1 item of a
// matrix sums the partials in a fixed order (deterministic norm) and
// publishes it with a release store.  Pass-2 items are queued after every
// pass-1 item of their matrix, so a waiting CTA only ever waits on CTAs that
// have claimed work ahead of it; the wait is still bounded and reports
// MUON_ERR_TIMEOUT instead of hanging.
#include "internal.h"
#include "ptx.cuh"

namespace muon {

namespace {


// L2 residency hints.  Pass 1 loads g and buf and stores buf with an
// evict-last policy: pass 2 of the same matrix reads them again a few
// hundred work items later, and the hint keeps more of them in L2 until
// then.  Pass 2 reads them for the last time, and writes X0 (which the next
// kernel reads only after every matrix is done), with an evict-first policy.
// (Measured: about 5% faster than without hints; outputs are unchanged.)
__device__ __forceinline__ uint64_t policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ float4 ld_hint(const float* a, uint64_t pol) {
  float4 v;
  asm volatile("ld.global.L2::cache_hint.v4.f32 {%0, %1, %2, %3}, [%4], %5;"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "l"(a), "l"(pol));
  return v;
}
__device__ __forceinline__ void st_hint(float* a, float4 v, uint64_t pol) {
  asm volatile("st.global.L2::cache_hint.v4.f32 [%0], {%1, %2, %3, %4}, %5;"
               :: "l"(a), "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w), "l"(pol) : "memory");
}

__device__ __forceinline__ void st_hint_u2(void* a, uint2 v, uint64_t pol) {
  asm volatile("st.global.L2::cache_hint.v2.b32 [%0], {%1, %2}, %3;"
               :: "l"(a), "r"(v.x), "r"(v.y), "l"(pol) : "memory");
}
__device__ __forceinline__ void st_hint_u4(void* a, uint4 v, uint64_t pol) {
  asm volatile("st.global.L2::cache_hint.v4.b32 [%0], {%1, %2, %3, %4}, %5;"
               :: "l"(a), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w), "l"(pol) : "memory");
}

__device__ __forceinline__ double block_sum(double v, double* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  __syncthreads();  // red may still be read by the previous call
  if (lane == 0) red[warp] = v;
  __syncthreads();
  double t = 0.0;
  if (threadIdx.x == 0) {
    for (int w = 0; w < K1_THREADS / 32; ++w) t += red[w];   // fixed order
  }
  return t;  // valid in thread 0 only
}

__device__ __forceinline__ float momentum_u(float g, float& b, float beta, int mode, int nesterov) {
  if (mode == K1_PLAIN) return g;
  b = fmaf(beta, b, g);
  return nesterov ? fmaf(beta, b, g) : b;
}

__device__ __forceinline__ float u_from(float g, float bnew, float beta, int mode, int nesterov) {
  if (mode == K1_PLAIN) return g;
  return nesterov ? fmaf(beta, bnew, g) : bnew;
}

// Pass 1 on one 64 x 64 tile: momentum (buf written back) and this thread's
// sum of squares of u.  Every load of the thread is issued before any store.
__device__ __forceinline__ double pass1_tile(const K1Launch& L, const K1Ptrs& P, long long r,
                                             long long c, long long r0, long long c0, int lrow,
                                             int lcol, uint64_t pol) {
  const bool vec = (c & 3) == 0;
  const float beta = L.beta;
  double ss = 0.0;
  float4 g4[4], b4[4];
  bool full[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const long long gr = r0 + lrow + 16 * k;
    const long long gc = c0 + lcol;
    full[k] = vec && gr < r && gc + 4 <= c;
    g4[k] = make_float4(0.f, 0.f, 0.f, 0.f);
    b4[k] = g4[k];
    if (full[k]) {
      const long long off = gr * c + gc;
      g4[k] = ld_hint(P.g + off, pol);
      if (L.mode != K1_PLAIN) b4[k] = ld_hint(P.buf + off, pol);
    }
  }
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const long long gr = r0 + lrow + 16 * k;
    const long long gc = c0 + lcol;
    if (full[k]) {
      float gv[4] = {g4[k].x, g4[k].y, g4[k].z, g4[k].w};
      float bv[4] = {b4[k].x, b4[k].y, b4[k].z, b4[k].w};
      float sq = 0.f;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float u = momentum_u(gv[e], bv[e], beta, L.mode, L.nesterov);
        sq = fmaf(u, u, sq);
      }
      ss += (double)sq;
      if (L.mode != K1_PLAIN)
        st_hint(P.buf + gr * c + gc, make_float4(bv[0], bv[1], bv[2], bv[3]), pol);
    } else if (gr < r && gc < c) {
      const long long off = gr * c + gc;
      for (int e = 0; e < 4 && gc + e < c; ++e) {
        float b = (L.mode != K1_PLAIN) ? P.buf[off + e] : 0.f;
        const float u = momentum_u(P.g[off + e], b, beta, L.mode, L.nesterov);
        ss += (double)u * (double)u;
        if (L.mode != K1_PLAIN) P.buf[off + e] = b;
      }
    }
  }
  return ss;
}

// Pass 2 on one 64 x 64 tile: recompute u from g and the new buf, scale by
// 1/(norm + eps) in double, round once to bf16 and store oriented.
__device__ __forceinline__ void pass2_tile(const K1Launch& L, const K1Ptrs& P, const K1Info& info,
                                           long long r0, long long c0, double inv, int tid,
                                           int lrow, int lcol, uint16_t (*s_tile)[K1_TILE + 2],
                                           uint64_t pol) {
  const long long r = info.r, c = info.c;
  const bool vec = (c & 3) == 0;
  const float beta = L.beta;
  const bool tr = info.transposed != 0;
  float4 g4[4], b4[4];
  bool full[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const long long gr = r0 + lrow + 16 * k;
    const long long gc = c0 + lcol;
    full[k] = vec && gr < r && gc + 4 <= c;
    g4[k] = make_float4(0.f, 0.f, 0.f, 0.f);
    b4[k] = g4[k];
    if (full[k]) {
      const long long off = gr * c + gc;
      g4[k] = ld_hint(P.g + off, pol);
      if (L.mode != K1_PLAIN) b4[k] = ld_hint(P.buf + off, pol);
    }
  }
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int row = lrow + 16 * k;
    const long long gr = r0 + row;
    const long long gc = c0 + lcol;
    uint16_t bits[4] = {0, 0, 0, 0};
    if (gr < r && gc < c) {
      const long long off = gr * c + gc;
      if (full[k]) {
        const float gv[4] = {g4[k].x, g4[k].y, g4[k].z, g4[k].w};
        const float bv[4] = {b4[k].x, b4[k].y, b4[k].z, b4[k].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float u = u_from(gv[e], bv[e], beta, L.mode, L.nesterov);
          bits[e] = __bfloat16_as_ushort(__double2bfloat16((double)u * inv));
        }
      } else {
        for (int e = 0; e < 4 && gc + e < c; ++e) {
          const float b = (L.mode != K1_PLAIN) ? __ldcg(P.buf + off + e) : 0.f;
          const float u = u_from(P.g[off + e], b, beta, L.mode, L.nesterov);
          bits[e] = __bfloat16_as_ushort(__double2bfloat16((double)u * inv));
        }
      }
      if (!tr) {
        __nv_bfloat16* dst = P.x0 + gr * info.ldx + gc;
        if (gc + 4 <= c) {
          uint2 w;
          w.x = (uint32_t)bits[0] | ((uint32_t)bits[1] << 16);
          w.y = (uint32_t)bits[2] | ((uint32_t)bits[3] << 16);
          st_hint_u2(dst, w, pol);
        } else {
          for (int e = 0; e < 4 && gc + e < c; ++e) dst[e] = __ushort_as_bfloat16(bits[e]);
        }
      }
    }
    if (tr) {
#pragma unroll
      for (int e = 0; e < 4; ++e) s_tile[row][lcol + e] = bits[e];
    }
  }
  if (tr) {
    __syncthreads();
    // X0 row (c0 + oc) holds stored column c0 + oc; 8 threads per row.
#pragma unroll
    for (int k2 = 0; k2 < 2; ++k2) {
      const int oc = (tid >> 3) + 32 * k2;
      const int seg = (tid & 7) * 8;
      const long long xr = c0 + oc;     // row of X0 (= stored column)
      const long long xc = r0 + seg;    // first column of X0 (= stored row)
      if (xr >= c || xc >= r) continue;
      __nv_bfloat16* dst = P.x0 + xr * info.ldx + xc;
      if (xc + 8 <= r) {
        uint4 w;
        w.x = (uint32_t)s_tile[seg + 0][oc] | ((uint32_t)s_tile[seg + 1][oc] << 16);
        w.y = (uint32_t)s_tile[seg + 2][oc] | ((uint32_t)s_tile[seg + 3][oc] << 16);
        w.z = (uint32_t)s_tile[seg + 4][oc] | ((uint32_t)s_tile[seg + 5][oc] << 16);
        w.w = (uint32_t)s_tile[seg + 6][oc] | ((uint32_t)s_tile[seg + 7][oc] << 16);
        st_hint_u4(dst, w, pol);
      } else {
        for (int e = 0; e < 8 && xc + e < r; ++e) dst[e] = __ushort_as_bfloat16(s_tile[seg + e][oc]);
      }
    }
    __syncthreads();   // s_tile is rewritten by the next tile
  }
}

__global__ void __launch_bounds__(K1_THREADS, 4) k1_kernel(const __grid_constant__ K1Launch L) {
  __shared__ int s_item;
  __shared__ int s_flag;
  __shared__ double s_norm;
  __shared__ double s_red[K1_THREADS / 32];
  __shared__ uint16_t s_tile[K1_TILE][K1_TILE + 2];

  const int tid = threadIdx.x;
  const uint64_t pol_keep = policy_evict_last();
  const uint64_t pol_drop = policy_evict_first();
  const int lrow = tid >> 4;         // 0..15
  const int lcol = (tid & 15) * 4;   // 0..60

  for (;;) {
    if (tid == 0) s_item = atomicAdd(L.counter, 1);
    __syncthreads();
    const int it = s_item;
    __syncthreads();
    if (it >= L.nitems) break;
    const K1Item item = L.items[it];
    const bool pass2 = (item.mat & K1_PASS2) != 0;
    const int mat = item.mat & ~K1_PASS2;
    if (kBoundsCheck) {
      // Checked builds: the item must name a matrix of the launch and one of
      // its groups, whose partial sum lies inside the partials array.
      bool ok = mat >= 0 && mat < L.n;
      if (ok) {
        const K1Info& q = L.info[mat];
        ok = item.group >= 0 && item.group < q.nitems && q.part0 >= 0 &&
             (long long)q.part0 + q.nitems <= L.npartials;
      }
      if (!ok) {
        if (tid == 0) atomicCAS(L.status, 0, MUON_ERR_INVALID_ARG);
        continue;
      }
    }
    const K1Info info = L.info[mat];
    const K1Ptrs P = L.ptrs[mat];
    const int t0 = item.group * K1_GROUP;
    const int t1 = min(t0 + K1_GROUP, info.ntiles);

    if (!pass2) {
      double ss = 0.0;
      for (int t = t0; t < t1; ++t) {
        const long long r0 = (long long)(t / info.tiles_c) * K1_TILE;
        const long long c0 = (long long)(t % info.tiles_c) * K1_TILE;
        ss += pass1_tile(L, P, info.r, info.c, r0, c0, lrow, lcol, pol_keep);
      }
      const double tot = block_sum(ss, s_red);
      if (tid == 0) {
        L.partials[info.part0 + item.group] = tot;
        // Release: this CTA's buf stores (ordered before by the barriers in
        // block_sum) and the partial become visible before the count does.
        __threadfence();
        const int prev = atomicAdd(L.done + mat, 1);
        s_flag = (prev == info.nitems - 1);
      }
      __syncthreads();
      if (s_flag) {
        // Last item of this matrix: fixed-order sum of its partials.
        __threadfence();
        double acc = 0.0;
        for (int t = tid; t < info.nitems; t += K1_THREADS) acc += __ldcg(L.partials + info.part0 + t);
        const double all = block_sum(acc, s_red);
        if (tid == 0) {
          L.norms[mat] = sqrt(all);
          __threadfence();
          st_release_gpu(L.ready + mat, 1);
        }
      }
      continue;
    }

    // ---------------------------------------------------------------- pass 2
    if (tid == 0) {
      int ok = ld_acquire_gpu(L.ready + mat);
      if (!ok) {
        const uint64_t t0ns = global_timer_ns();
        while (!(ok = ld_acquire_gpu(L.ready + mat))) {
          if (global_timer_ns() - t0ns > L.limit_ns) break;
          __nanosleep(128);
        }
      }
      if (!ok) atomicCAS(L.status, 0, MUON_ERR_TIMEOUT);
      s_flag = ok;
      s_norm = ok ? __ldcg(L.norms + mat) : 0.0;
    }
    __syncthreads();
    if (!s_flag) continue;
    const double inv = 1.0 / (s_norm + 1e-7);
    for (int t = t0; t < t1; ++t) {
      const long long r0 = (long long)(t / info.tiles_c) * K1_TILE;
      const long long c0 = (long long)(t % info.tiles_c) * K1_TILE;
      pass2_tile(L, P, info, r0, c0, inv, tid, lrow, lcol, s_tile, pol_drop);
    }
  }
}

// p <- p - scale * X0 (or a plain copy of X0 out) for ns_steps == 0.
__global__ void apply_kernel(const __grid_constant__ ApplyLaunch L) {
  const int mat = blockIdx.y;
  if (mat >= L.n) return;
  const K1Info info = L.info[mat];
  const long long r = info.r, c = info.c, total = r * c;
  const __nv_bfloat16* x0 = L.ptrs[mat].x0;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (long long)gridDim.x * blockDim.x) {
    const long long i = e / c, j = e % c;                 // stored position
    const long long xo = info.transposed ? (j * info.ldx + i) : (i * info.ldx + j);
    const float x = __bfloat162float(x0[xo]);
    if (L.mode == FINAL_PARAM) {
      float* p = reinterpret_cast<float*>(L.dst[mat]) + e;
      *p = __fadd_rn(*p, __fmul_rn(-L.scale[mat], x));   // p + fp32(-s x), as the GEMM paths
    } else if (L.mode == FINAL_OUT_F32) {
      reinterpret_cast<float*>(L.dst[mat])[e] = x;
    } else {
      reinterpret_cast<__nv_bfloat16*>(L.dst[mat])[e] = __float2bfloat16_rn(x);
    }
  }
}

}  // namespace

int k1_blocks_per_sm() {
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k1_kernel, K1_THREADS, 0) != cudaSuccess || n < 1)
    return 1;
  return n;
}

cudaError_t launch_k1(const K1Launch& L, int grid, cudaStream_t stream) {
  if (L.nitems <= 0) return cudaSuccess;
  k1_kernel<<<grid, K1_THREADS, 0, stream>>>(L);
  return cudaGetLastError();
}

cudaError_t launch_apply(const ApplyLaunch& L, cudaStream_t stream) {
  if (L.n <= 0) return cudaSuccess;
  apply_kernel<<<dim3(256, L.n), 256, 0, stream>>>(L);
  return cudaGetLastError();
}

}  // namespace muon
