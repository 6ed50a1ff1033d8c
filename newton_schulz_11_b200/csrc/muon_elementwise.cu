// Elementwise stage of the Muon step, HBM-bound.
//
//   m' = beta m + g                        ("14 - modded-nanogpt", section 3, muon_step)
//   u  = g + beta m'  (Nesterov) or m'     ("NanoGPT Speedrun" README, practices list)
//   hi = bf16(u), lo = 8-bit residual      Newton-Schulz input, unscaled (lo: the byte
//                                          (bits(u) - bits(hi) + 2^15 + 2^8) >> 9, so that
//                                          u ~ the float with bits bits(hi) + 2^9 (lo - 64))
//   partial[chunk] = sum of u^2            for ||u||_F of the listing's G.norm()
//   non-finite u                           counted into the workspace header, which then
//                                          reports MUON_ERR_NONFINITE (values propagate)
//
// Rows whose length is a multiple of 8 are read and written eight elements at a time
// (256-bit accesses on 32-byte aligned rows, two 128-bit ones on 16-byte aligned rows,
// the same element order either way); other rows four at a time, or one by one.
// followed by a per-matrix finalisation s = 1 / (||u||_F + eps) in a fixed order
// (deterministic: no atomics).  One CTA handles one chunk of whole rows of one
// matrix; rows are read with 128-bit loads when the layout allows it.
#include "muon_device.cuh"
#include "muon_params.h"

namespace muon {

constexpr int kEwThreads = 256;

__device__ __forceinline__ float block_sum(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float s = 0.f;
  if (warp == 0) {
    s = lane < (kEwThreads / 32) ? red[lane] : 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  }
  return s;  // valid in thread 0
}

__device__ __forceinline__ int find_matrix(const EwParams& p, int chunk) {
  int lo = 0, hi = p.n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (p.mats[mid].chunk_begin <= chunk) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__device__ __forceinline__ float ew_one(float g, float& m, float beta, int nesterov, int ns_only) {
  if (ns_only) return g;
  const float mn = fmaf(beta, m, g);
  m = mn;
  return nesterov ? fmaf(beta, mn, g) : mn;
}

__global__ void __launch_bounds__(kEwThreads) muon_momentum_kernel(const __grid_constant__ EwParams p) {
  __shared__ float red[kEwThreads / 32];
  griddep_launch_dependents();
  griddep_wait();  // the previous step may still read the hi/lo buffers this writes
  const int chunk = blockIdx.x;
  const int i = find_matrix(p, chunk);
  const EwMat& t = p.mats[i];
  const int r0 = (chunk - t.chunk_begin) * t.rows_per_chunk;
  const int r1 = min(t.rows, r0 + t.rows_per_chunk);
  const float beta = p.beta;
  const int nesterov = p.nesterov, ns_only = p.ns_only;
  float acc = 0.f;
  int nf = 0;  // non-finite values of u seen by this thread

  if (t.vec >= 2) {
    // eight elements per thread and iteration: one 256-bit access per row segment where
    // the rows are 32-byte aligned (vec 2), two 128-bit ones where they are 16-byte
    // aligned (vec 3); both visit the elements in the same order, so the sums of squares
    // and everything after them do not depend on the alignment
    const bool v8 = t.vec == 2;
    const int c8 = t.cols >> 3;
    const int total = (r1 - r0) * c8;
    for (int idx = threadIdx.x; idx < total; idx += kEwThreads) {
      const int rr = idx / c8;
      const int c = (idx - rr * c8) << 3;
      const int r = r0 + rr;
      const float* gp = t.g + static_cast<int64_t>(r) * t.ld_g + c;
      float* mp = t.m + static_cast<int64_t>(r) * t.ld_m + c;
      float g[8], m[8], u[8];
      if (v8) {
        ld_global_cs_v8(gp, g);
      } else {
        const float4 g0 = __ldcs(reinterpret_cast<const float4*>(gp)), g1 = __ldcs(reinterpret_cast<const float4*>(gp) + 1);
        g[0] = g0.x, g[1] = g0.y, g[2] = g0.z, g[3] = g0.w, g[4] = g1.x, g[5] = g1.y, g[6] = g1.z, g[7] = g1.w;
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) m[j] = 0.f;
      if (!ns_only) {
        if (v8) {
          ld_global_cs_v8(mp, m);
        } else {
          const float4 m0 = __ldcs(reinterpret_cast<const float4*>(mp)), m1 = __ldcs(reinterpret_cast<const float4*>(mp) + 1);
          m[0] = m0.x, m[1] = m0.y, m[2] = m0.z, m[3] = m0.w, m[4] = m1.x, m[5] = m1.y, m[6] = m1.z, m[7] = m1.w;
        }
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) u[j] = ew_one(g[j], m[j], beta, nesterov, ns_only);
      if (!ns_only) {
        if (v8) {
          st_global_cs_v8(mp, m);
        } else {
          __stcs(reinterpret_cast<float4*>(mp), make_float4(m[0], m[1], m[2], m[3]));
          __stcs(reinterpret_cast<float4*>(mp) + 1, make_float4(m[4], m[5], m[6], m[7]));
        }
      }
      uint32_t h01, h23, h45, h67, l0, l1;
      split_hi_lo8x4(u[0], u[1], u[2], u[3], h01, h23, l0);
      split_hi_lo8x4(u[4], u[5], u[6], u[7], h45, h67, l1);
      *reinterpret_cast<uint4*>(t.hi + static_cast<int64_t>(r) * t.ldx + c) = make_uint4(h01, h23, h45, h67);
      *reinterpret_cast<uint2*>(t.lo + static_cast<int64_t>(r) * t.ldl + c) = make_uint2(l0, l1);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        acc = fmaf(u[j], u[j], acc);
        nf += isfinite(u[j]) ? 0 : 1;
      }
    }
  } else if (t.vec) {
    const int c4 = t.cols >> 2;
    const int total = (r1 - r0) * c4;
    for (int idx = threadIdx.x; idx < total; idx += kEwThreads) {
      const int rr = idx / c4;
      const int c = (idx - rr * c4) << 2;
      const int r = r0 + rr;
      const float4 g = __ldcs(reinterpret_cast<const float4*>(t.g + static_cast<int64_t>(r) * t.ld_g + c));
      float4 m = make_float4(0.f, 0.f, 0.f, 0.f);
      float* mp = t.m + static_cast<int64_t>(r) * t.ld_m + c;
      if (!ns_only) m = __ldcs(reinterpret_cast<const float4*>(mp));
      float u0 = ew_one(g.x, m.x, beta, nesterov, ns_only);
      float u1 = ew_one(g.y, m.y, beta, nesterov, ns_only);
      float u2 = ew_one(g.z, m.z, beta, nesterov, ns_only);
      float u3 = ew_one(g.w, m.w, beta, nesterov, ns_only);
      if (!ns_only) __stcs(reinterpret_cast<float4*>(mp), m);
      uint32_t h01, h23, l4;
      split_hi_lo8x4(u0, u1, u2, u3, h01, h23, l4);
      *reinterpret_cast<uint2*>(t.hi + static_cast<int64_t>(r) * t.ldx + c) = make_uint2(h01, h23);
      *reinterpret_cast<uint32_t*>(t.lo + static_cast<int64_t>(r) * t.ldl + c) = l4;
      acc = fmaf(u0, u0, acc);
      acc = fmaf(u1, u1, acc);
      acc = fmaf(u2, u2, acc);
      acc = fmaf(u3, u3, acc);
      nf += (isfinite(u0) ? 0 : 1) + (isfinite(u1) ? 0 : 1) + (isfinite(u2) ? 0 : 1) + (isfinite(u3) ? 0 : 1);
    }
  } else {
    const int total = (r1 - r0) * t.cols;
    for (int idx = threadIdx.x; idx < total; idx += kEwThreads) {
      const int rr = idx / t.cols;
      const int c = idx - rr * t.cols;
      const int r = r0 + rr;
      const float g = t.g[static_cast<int64_t>(r) * t.ld_g + c];
      float* mp = t.m + static_cast<int64_t>(r) * t.ld_m + c;
      float m = ns_only ? 0.f : *mp;
      const float u = ew_one(g, m, beta, nesterov, ns_only);
      if (!ns_only) *mp = m;
      const uint32_t h = float_to_bf16_bits(u);
      t.hi[static_cast<int64_t>(r) * t.ldx + c] = __ushort_as_bfloat16(static_cast<unsigned short>(h));
      t.lo[static_cast<int64_t>(r) * t.ldl + c] = static_cast<uint8_t>(lo8_encode(u, h));
      acc = fmaf(u, u, acc);
      nf += isfinite(u) ? 0 : 1;
    }
  }
  const float s = block_sum(acc, red);
  if (threadIdx.x == 0) p.partials[chunk] = s;
  if (__syncthreads_or(nf != 0)) {  // rare: this chunk holds a NaN or an infinity
    const int w = __reduce_add_sync(0xffffffffu, nf);
    if ((threadIdx.x & 31) == 0 && w != 0)
      atomicAdd(reinterpret_cast<unsigned long long*>(p.status + 2), static_cast<unsigned long long>(w));
    if (threadIdx.x == 0 && atomicCAS(&p.status[0], 0, kStatusNonfinite) == 0) atomicExch(&p.status[1], t.index);
  }
}

// s_i = 1 / (sqrt(sum of the matrix's chunk partials) + eps), summed in fp64 in a
// fixed order.
__global__ void __launch_bounds__(kEwThreads) muon_norm_kernel(const __grid_constant__ EwParams p) {
  __shared__ double red[kEwThreads];
  griddep_launch_dependents();
  griddep_wait();
  const EwMat& t = p.mats[blockIdx.x];
  double s = 0.0;
  for (int k = threadIdx.x; k < t.nchunks; k += kEwThreads) s += static_cast<double>(p.partials[t.chunk_begin + k]);
  red[threadIdx.x] = s;
  __syncthreads();
  for (int w = kEwThreads / 2; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    const double nrm = sqrt(red[0]);
    p.norm[blockIdx.x] = static_cast<float>(nrm);
    p.scale[blockIdx.x] = static_cast<float>(1.0 / (nrm + static_cast<double>(p.eps)));
  }
}

template <typename K>
static cudaError_t launch_pdl(K kernel, int grid, const EwParams& p, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(kEwThreads, 1, 1);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, p);
}

cudaError_t launch_momentum(const EwParams& p, cudaStream_t stream) {
  return launch_pdl(muon_momentum_kernel, p.total_chunks, p, stream);
}

cudaError_t launch_norm(const EwParams& p, cudaStream_t stream) { return launch_pdl(muon_norm_kernel, p.n, p, stream); }

}  // namespace muon
