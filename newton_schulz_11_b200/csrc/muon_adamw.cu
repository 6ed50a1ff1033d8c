// AdamW for the parameters Muon does not take: the 1-D parameters (biases, norm gains)
// and the embeddings ("14 - modded-nanogpt: the Speedrun Community", section 3: the
// canonical setup is hybrid, Muon on the 2-D matmul weights and AdamW on the rest).
// The pages give no formula; this is the textbook decoupled-decay AdamW with bias
// correction, in the form PyTorch uses:
//
//   m <- beta1 m + (1 - beta1) g
//   v <- beta2 v + (1 - beta2) g^2
//   p <- p (1 - lr wd) - (lr / (1 - beta1^t)) m / (sqrt(v) / sqrt(1 - beta2^t) + eps)
//
// One fused, HBM-bound pass over a grouped list of flattened tensors: each CTA takes a
// chunk of one tensor, 128-bit streaming loads and stores where every pointer allows it,
// fp32 arithmetic, round-to-nearest-even into a bf16 parameter.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <vector>

#include "muon_b200.h"
#include "muon_device.cuh"

namespace muon {

constexpr int kAdamThreads = 256;
constexpr int64_t kAdamChunk = 16384;  // elements per CTA (a multiple of 4)
constexpr int kAdamMaxTensors = 128;   // per launch

struct AdamTensor {
  void* p;
  const float* g;
  float* m;
  float* v;
  int64_t numel;
  int64_t chunk_begin;  // first chunk of this tensor in the launch
  int32_t p_bf16;
  int32_t vec;  // 1: 16-byte aligned g, m, v (p: 8 bytes for bf16, 16 for fp32); 2: twice that
};

struct AdamParams {
  AdamTensor t[kAdamMaxTensors];
  int32_t n;
  float beta1, beta2, omb1, omb2, eps;
  float decay;         // 1 - lr wd
  float step_size;     // lr / (1 - beta1^t)
  float inv_sqrt_bc2;  // 1 / sqrt(1 - beta2^t)
};

__device__ __forceinline__ int find_tensor(const AdamParams& p, int64_t chunk) {
  int lo = 0, hi = p.n - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (p.t[mid].chunk_begin <= chunk) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// One element: updates m and v in place and returns the new parameter value.
__device__ __forceinline__ float adam_one(const AdamParams& a, float pv, float g, float& m, float& v) {
  m = fmaf(a.beta1, m, a.omb1 * g);
  v = fmaf(a.beta2, v, a.omb2 * (g * g));
  const float denom = sqrtf(v) * a.inv_sqrt_bc2 + a.eps;
  return fmaf(pv, a.decay, -(a.step_size * (m / denom)));
}

__global__ void __launch_bounds__(kAdamThreads) muon_adamw_kernel(const __grid_constant__ AdamParams a) {
  const int64_t chunk = blockIdx.x;
  const AdamTensor& t = a.t[find_tensor(a, chunk)];
  const int64_t e0 = (chunk - t.chunk_begin) * kAdamChunk;
  const int64_t e1 = t.numel < e0 + kAdamChunk ? t.numel : e0 + kAdamChunk;
  int64_t scalar_from = e0;
  if (t.vec == 2) {  // 32-byte aligned tensors: eight elements per thread and access
    const int64_t n8 = (e1 - e0) >> 3;
    for (int64_t i = threadIdx.x; i < n8; i += kAdamThreads) {
      const int64_t e = e0 + 8 * i;
      float g[8], m[8], v[8], pv[8];
      ld_global_cs_v8(t.g + e, g);
      ld_global_cs_v8(t.m + e, m);
      ld_global_cs_v8(t.v + e, v);
      if (t.p_bf16) {
        __nv_bfloat16* pp = static_cast<__nv_bfloat16*>(t.p) + e;
        const uint4 raw = __ldcs(reinterpret_cast<const uint4*>(pp));
        const uint32_t rw[4] = {raw.x, raw.y, raw.z, raw.w};
        uint32_t out[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float p0 = adam_one(a, bf16_bits_to_float(rw[k] & 0xFFFFu), g[2 * k], m[2 * k], v[2 * k]);
          const float p1 = adam_one(a, bf16_bits_to_float(rw[k] >> 16), g[2 * k + 1], m[2 * k + 1], v[2 * k + 1]);
          const __nv_bfloat162 q = __floats2bfloat162_rn(p0, p1);
          out[k] = *reinterpret_cast<const uint32_t*>(&q);
        }
        __stcs(reinterpret_cast<uint4*>(pp), make_uint4(out[0], out[1], out[2], out[3]));
      } else {
        float* pp = static_cast<float*>(t.p) + e;
        ld_global_cs_v8(pp, pv);
#pragma unroll
        for (int k = 0; k < 8; ++k) pv[k] = adam_one(a, pv[k], g[k], m[k], v[k]);
        st_global_cs_v8(pp, pv);
      }
      st_global_cs_v8(t.m + e, m);
      st_global_cs_v8(t.v + e, v);
    }
    scalar_from = e0 + 8 * n8;
  } else if (t.vec) {
    const int64_t n4 = (e1 - e0) >> 2;
    for (int64_t i = threadIdx.x; i < n4; i += kAdamThreads) {
      const int64_t e = e0 + 4 * i;
      const float4 g = __ldcs(reinterpret_cast<const float4*>(t.g + e));
      float4 m = __ldcs(reinterpret_cast<const float4*>(t.m + e));
      float4 v = __ldcs(reinterpret_cast<const float4*>(t.v + e));
      if (t.p_bf16) {
        __nv_bfloat16* pp = static_cast<__nv_bfloat16*>(t.p) + e;
        const uint2 raw = __ldcs(reinterpret_cast<const uint2*>(pp));
        const float p0 = adam_one(a, bf16_bits_to_float(raw.x & 0xFFFFu), g.x, m.x, v.x);
        const float p1 = adam_one(a, bf16_bits_to_float(raw.x >> 16), g.y, m.y, v.y);
        const float p2 = adam_one(a, bf16_bits_to_float(raw.y & 0xFFFFu), g.z, m.z, v.z);
        const float p3 = adam_one(a, bf16_bits_to_float(raw.y >> 16), g.w, m.w, v.w);
        const __nv_bfloat162 q0 = __floats2bfloat162_rn(p0, p1), q1 = __floats2bfloat162_rn(p2, p3);
        __stcs(reinterpret_cast<uint2*>(pp), make_uint2(*reinterpret_cast<const uint32_t*>(&q0),
                                                         *reinterpret_cast<const uint32_t*>(&q1)));
      } else {
        float* pp = static_cast<float*>(t.p) + e;
        float4 pv = __ldcs(reinterpret_cast<const float4*>(pp));
        pv.x = adam_one(a, pv.x, g.x, m.x, v.x);
        pv.y = adam_one(a, pv.y, g.y, m.y, v.y);
        pv.z = adam_one(a, pv.z, g.z, m.z, v.z);
        pv.w = adam_one(a, pv.w, g.w, m.w, v.w);
        __stcs(reinterpret_cast<float4*>(pp), pv);
      }
      __stcs(reinterpret_cast<float4*>(t.m + e), m);
      __stcs(reinterpret_cast<float4*>(t.v + e), v);
    }
    scalar_from = e0 + 4 * n4;
  }
  for (int64_t e = scalar_from + threadIdx.x; e < e1; e += kAdamThreads) {
    float m = t.m[e], v = t.v[e];
    if (t.p_bf16) {
      __nv_bfloat16* pp = static_cast<__nv_bfloat16*>(t.p) + e;
      const float pn = adam_one(a, bf16_bits_to_float(__bfloat16_as_ushort(*pp)), t.g[e], m, v);
      *pp = __float2bfloat16_rn(pn);
    } else {
      float* pp = static_cast<float*>(t.p) + e;
      *pp = adam_one(a, *pp, t.g[e], m, v);
    }
    t.m[e] = m;
    t.v[e] = v;
  }
}

}  // namespace muon

// ---------------------------------------------------------------- host side

namespace {

using muon::AdamParams;

bool aligned_to(const void* p, size_t a) { return reinterpret_cast<uintptr_t>(p) % a == 0; }

struct Range {
  uintptr_t lo, hi;
  bool write;
};

// Every buffer the call writes (param, exp_avg, exp_avg_sq) must overlap no other buffer
// of the call; gradients are only read and may overlap one another.
bool ranges_disjoint(std::vector<Range>& r) {
  std::sort(r.begin(), r.end(), [](const Range& a, const Range& b) { return a.lo < b.lo; });
  uintptr_t max_hi = 0;
  bool max_write = false;
  for (size_t i = 0; i < r.size(); ++i) {
    if (i > 0 && r[i].lo < max_hi && (r[i].write || max_write)) return false;
    if (r[i].hi > max_hi) {
      max_hi = r[i].hi;
      max_write = r[i].write;
    } else if (r[i].write) {
      return false;  // inside an earlier range
    }
  }
  return true;
}

muon_status_t adamw_device_ok() {
  int dev = 0, major = 0, minor = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MUON_ERR_NO_DEVICE;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return MUON_ERR_CUDA;
  return (major == 10 && minor == 0) ? MUON_OK : MUON_ERR_NO_DEVICE;
}

}  // namespace

extern "C" muon_status_t muon_adamw_step(const muon_adamw_tensor_t* ts, int n, float lr, float beta1, float beta2,
                                         float eps, float weight_decay, int64_t step, void* stream) {
  if (ts == nullptr || n < 1) return MUON_ERR_INVALID_ARG;
  if (!std::isfinite(lr) || !std::isfinite(beta1) || !std::isfinite(beta2) || !std::isfinite(eps) ||
      !std::isfinite(weight_decay) || lr < 0.f || beta1 < 0.f || beta1 >= 1.f || beta2 < 0.f || beta2 >= 1.f ||
      !(eps > 0.f) || weight_decay < 0.f || step < 1)
    return MUON_ERR_INVALID_ARG;
  std::vector<Range> ranges;
  ranges.reserve(4 * static_cast<size_t>(n));
  for (int i = 0; i < n; ++i) {
    const muon_adamw_tensor_t& t = ts[i];
    if (t.param == nullptr || t.grad == nullptr || t.exp_avg == nullptr || t.exp_avg_sq == nullptr)
      return MUON_ERR_INVALID_ARG;
    if (t.numel < 1) return MUON_ERR_UNSUPPORTED_SHAPE;
    if (t.param_dtype != MUON_F32 && t.param_dtype != MUON_BF16) return MUON_ERR_UNSUPPORTED_DTYPE;
    const size_t pb = t.param_dtype == MUON_BF16 ? 2 : 4;
    if (!aligned_to(t.param, pb) || !aligned_to(t.grad, 4) || !aligned_to(t.exp_avg, 4) ||
        !aligned_to(t.exp_avg_sq, 4))
      return MUON_ERR_ALIGNMENT;
    const uintptr_t nb = static_cast<uintptr_t>(t.numel);
    ranges.push_back({reinterpret_cast<uintptr_t>(t.param), reinterpret_cast<uintptr_t>(t.param) + nb * pb, true});
    ranges.push_back({reinterpret_cast<uintptr_t>(t.exp_avg), reinterpret_cast<uintptr_t>(t.exp_avg) + nb * 4, true});
    ranges.push_back(
        {reinterpret_cast<uintptr_t>(t.exp_avg_sq), reinterpret_cast<uintptr_t>(t.exp_avg_sq) + nb * 4, true});
    ranges.push_back({reinterpret_cast<uintptr_t>(t.grad), reinterpret_cast<uintptr_t>(t.grad) + nb * 4, false});
  }
  if (!ranges_disjoint(ranges)) return MUON_ERR_INVALID_ARG;
  muon_status_t st = adamw_device_ok();
  if (st != MUON_OK) return st;

  AdamParams a{};
  a.beta1 = beta1;
  a.beta2 = beta2;
  a.omb1 = 1.f - beta1;
  a.omb2 = 1.f - beta2;
  a.eps = eps;
  a.decay = 1.f - lr * weight_decay;
  const double bc1 = 1.0 - std::pow(static_cast<double>(beta1), static_cast<double>(step));
  const double bc2 = 1.0 - std::pow(static_cast<double>(beta2), static_cast<double>(step));
  a.step_size = static_cast<float>(static_cast<double>(lr) / bc1);
  a.inv_sqrt_bc2 = static_cast<float>(1.0 / std::sqrt(bc2));
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  for (int base = 0; base < n; base += muon::kAdamMaxTensors) {
    const int cnt = std::min(muon::kAdamMaxTensors, n - base);
    int64_t chunks = 0;
    for (int k = 0; k < cnt; ++k) {
      const muon_adamw_tensor_t& t = ts[base + k];
      muon::AdamTensor& d = a.t[k];
      d.p = t.param;
      d.g = t.grad;
      d.m = t.exp_avg;
      d.v = t.exp_avg_sq;
      d.numel = t.numel;
      d.chunk_begin = chunks;
      d.p_bf16 = t.param_dtype == MUON_BF16 ? 1 : 0;
      d.vec = (aligned_to(t.grad, 32) && aligned_to(t.exp_avg, 32) && aligned_to(t.exp_avg_sq, 32) &&
               aligned_to(t.param, d.p_bf16 ? 16 : 32))
                  ? 2
              : (aligned_to(t.grad, 16) && aligned_to(t.exp_avg, 16) && aligned_to(t.exp_avg_sq, 16) &&
                 aligned_to(t.param, d.p_bf16 ? 8 : 16))
                  ? 1
                  : 0;
      chunks += (t.numel + muon::kAdamChunk - 1) / muon::kAdamChunk;
    }
    a.n = cnt;
    if (chunks > 0x7fffffff) return MUON_ERR_UNSUPPORTED_SHAPE;
    muon::muon_adamw_kernel<<<static_cast<unsigned>(chunks), muon::kAdamThreads, 0, s>>>(a);
    if (cudaGetLastError() != cudaSuccess) return MUON_ERR_CUDA;
  }
  return MUON_OK;
}
