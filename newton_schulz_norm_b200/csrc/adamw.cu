// adamw.cu -- one AdamW step over a list of fp32 tensors in a single launch.
//
// The GPT-2 parameters that the Muon step leaves out (embeddings, LayerNorm
// gains and biases, linear biases) take AdamW.  "07. Training neural
// networks", section "Adam, weight decay and AdamW", defines the step: two
// running averages per entry (of the gradient and of its square), bias
// correction by 1 - beta^t, the move lr * u_hat / (sqrt(v_hat) + eps), and
// decoupled decay that first multiplies the parameter by (1 - lr * lambda).
//
// The work is a stream: 16 bytes read and 12 bytes written per element, no
// reuse.  So the kernel is shaped for HBM bandwidth only: persistent CTAs
// (occupancy x SM count), chunks of 2048 elements handed out in grid-stride
// order across every tensor of the call, 16-byte vector loads issued for all
// four arrays before any arithmetic so that each thread keeps eight loads in
// flight, and cache-streaming hints since nothing is read twice.  Tensors
// whose pointers are not all 16-byte aligned take a scalar path with the
// same arithmetic.
#include "internal.h"

namespace muon {
namespace {

// One element, in the order the page gives the step.  fp32 throughout;
// sqrtf and the division are IEEE round-to-nearest (no fast-math).
__device__ __forceinline__ void adamw_elem(float& p, float g, float& m, float& v,
                                           const AdamWLaunch& L, float decay) {
  m = fmaf(L.beta1, m, L.one_minus_beta1 * g);
  v = fmaf(L.beta2, v, L.one_minus_beta2 * (g * g));
  const float den = fmaf(sqrtf(v), L.inv_sqrt_bc2, L.eps);   // sqrt(v_hat) + eps
  p = fmaf(p, decay, -(L.step_size * m) / den);              // decay, then the Adam move
}

__device__ __forceinline__ void scalar_elem(const AdamWTensor& T, long long e, const AdamWLaunch& L) {
  float p = __ldcs(T.p + e), g = __ldcs(T.g + e), m = __ldcs(T.m + e), v = __ldcs(T.v + e);
  adamw_elem(p, g, m, v, L, T.decay);
  __stcs(T.p + e, p);
  __stcs(T.m + e, m);
  __stcs(T.v + e, v);
}

__global__ void __launch_bounds__(ADAMW_THREADS, 4) adamw_kernel(const __grid_constant__ AdamWLaunch L) {
  int ti = 0;
  for (int c = blockIdx.x; c < L.nchunks; c += gridDim.x) {
    while (ti + 1 < L.n && L.t[ti + 1].chunk0 <= c) ++ti;   // chunks only grow
    const AdamWTensor& T = L.t[ti];
    const long long e0 = (long long)(c - T.chunk0) * ADAMW_CHUNK;
    const long long e1 = min(e0 + (long long)ADAMW_CHUNK, T.numel);
    if (T.vec) {
      const long long q0 = e0 >> 2, q1 = e1 >> 2;   // whole float4s of the chunk
      const float4* p4 = reinterpret_cast<const float4*>(T.p);
      const float4* g4 = reinterpret_cast<const float4*>(T.g);
      const float4* m4 = reinterpret_cast<const float4*>(T.m);
      const float4* v4 = reinterpret_cast<const float4*>(T.v);
      float4 p[ADAMW_VEC], g[ADAMW_VEC], m[ADAMW_VEC], v[ADAMW_VEC];
#pragma unroll
      for (int j = 0; j < ADAMW_VEC; ++j) {
        const long long q = q0 + threadIdx.x + (long long)j * ADAMW_THREADS;
        if (q < q1) {
          p[j] = __ldcs(p4 + q);
          g[j] = __ldcs(g4 + q);
          m[j] = __ldcs(m4 + q);
          v[j] = __ldcs(v4 + q);
        }
      }
#pragma unroll
      for (int j = 0; j < ADAMW_VEC; ++j) {
        const long long q = q0 + threadIdx.x + (long long)j * ADAMW_THREADS;
        if (q < q1) {
          adamw_elem(p[j].x, g[j].x, m[j].x, v[j].x, L, T.decay);
          adamw_elem(p[j].y, g[j].y, m[j].y, v[j].y, L, T.decay);
          adamw_elem(p[j].z, g[j].z, m[j].z, v[j].z, L, T.decay);
          adamw_elem(p[j].w, g[j].w, m[j].w, v[j].w, L, T.decay);
          __stcs(reinterpret_cast<float4*>(T.p) + q, p[j]);
          __stcs(reinterpret_cast<float4*>(T.m) + q, m[j]);
          __stcs(reinterpret_cast<float4*>(T.v) + q, v[j]);
        }
      }
      // the last chunk of a tensor whose length is not a multiple of 4
      const long long e = (q1 << 2) + threadIdx.x;
      if (e < e1) scalar_elem(T, e, L);
    } else {
      for (long long e = e0 + threadIdx.x; e < e1; e += ADAMW_THREADS) scalar_elem(T, e, L);
    }
  }
}

}  // namespace

int adamw_blocks_per_sm() {
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, adamw_kernel, ADAMW_THREADS, 0) != cudaSuccess ||
      n < 1)
    return 1;
  return n;
}

cudaError_t launch_adamw(const AdamWLaunch& L, int grid, cudaStream_t stream) {
  if (L.nchunks <= 0 || L.n <= 0) return cudaSuccess;
  adamw_kernel<<<grid, ADAMW_THREADS, 0, stream>>>(L);
  return cudaGetLastError();
}

}  // namespace muon
