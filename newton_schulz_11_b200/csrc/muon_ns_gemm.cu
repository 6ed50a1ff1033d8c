// Newton-Schulz contractions on the 5th-generation tensor cores (tcgen05, sm_100a).
//
// One persistent, warp-specialised kernel serves the three products of an iteration
// ("NanoGPT Speedrun" README, zeroth_power_via_newtonschulz5 listing, loop body):
//
//   kGram       A = X X^T                 (s^2 X X^T on iteration 0, X still unscaled)
//   kPoly       B = b A + c A A           (A symmetric, so A A = A A^T)
//   kApply      X <- s (a X + B X)        (s = 1 / (||u|| + eps) on iteration 0, else 1)
//   kApplyLast  same, then W <- W (1 - lr wd) - lr shape_scale X   and/or   O <- X
//
// The Gram and the polynomial are symmetric: only tiles that touch the upper
// triangle are computed, and each element (r <= c) is stored twice, at (r, c) and
// (c, r), by the one thread that owns it -- so every element has exactly one writer.
//
// A tall matrix (rows > cols) is never transposed in memory.  With Y the stored
// matrix (X = Y^T) the same iteration reads  A = Y^T Y  (both operands MN-major)
// and  Y <- a Y + Y B  (B symmetric), so the kernel takes operand majorness per
// shape class at run time.
//
// Roles (192 threads, one CTA per SM, persistent over a flat tile list):
//   warp 0      one thread issues TMA loads of 64x64 bf16 boxes (128-byte swizzle)
//               into a ring of shared-memory stages
//   warp 1      allocates TMEM (two fp32 accumulators of 128 x BN); one thread issues
//               tcgen05.mma (M = 128, N = BN, K = 16) and commits to mbarriers
//   warps 2..5  epilogue: tcgen05.ld of the accumulator (TMEM lane = tile row),
//               fused coefficient math, global stores
// The epilogue of tile t overlaps the main loop of tile t + 1.
#include "muon_device.cuh"
#include "muon_params.h"

namespace muon {

template <int BN>
struct GemmCfg {
  static constexpr int kABytes = kBM * kBK * 2;
  static constexpr int kBBytes = BN * kBK * 2;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kStages = BN == 256 ? 4 : 6;
  static constexpr int kTmemCols = 2 * BN;
  static constexpr int kBarrierBytes = 256;
  static constexpr int kSmemBytes = kStages * kStageBytes + 1024 + kBarrierBytes;
  static_assert(kStages * 2 + 5 <= kBarrierBytes / 8 - 2, "barrier area too small");
};

constexpr int kGemmThreads = 192;

// Waits on the way out (loads and MMAs already in flight) get at least two seconds,
// whatever the per-wait budget: they end by themselves, and leaving before they do
// would let a copy land in shared memory this CTA no longer owns.
__device__ __forceinline__ unsigned long long teardown_budget(unsigned long long budget) {
  return budget > 2000000000ull ? budget : 2000000000ull;
}

template <int MODE>
struct ParamsOf {
  using type = GemmParams;
};
template <>
struct ParamsOf<kApplyLast> {
  using type = FinalParams;
};

struct Tile {
  int cls, mat, ib, jb;
};

template <int MODE, int BN>
__device__ __forceinline__ Tile decode_tile(const GemmParams& p, int t) {
  int c = 0;
  while (c + 1 < p.num_classes && t >= p.cls[c + 1].tile_begin) ++c;
  const ClassDesc& cd = p.cls[c];
  const int local = t - cd.tile_begin;
  Tile r;
  r.cls = c;
  r.mat = local / cd.tiles_per_mat;
  int q = local - r.mat * cd.tiles_per_mat;
  if (MODE == kGram || MODE == kPoly) {
    // Row tile ib needs the column tiles from the one holding column ib * BM onwards.
    int ib = 0;
    for (;;) {
      const int first = (ib * kBM) / BN;
      const int cnt = cd.nb - first;
      if (q < cnt) {
        r.ib = ib;
        r.jb = first + q;
        break;
      }
      q -= cnt;
      ++ib;
    }
  } else if (cd.i_fast) {
    r.ib = q % cd.mb;
    r.jb = q / cd.mb;
  } else {
    r.jb = q % cd.nb;
    r.ib = q / cd.nb;
  }
  return r;
}

// One 64-row (K-major) or 64-column (MN-major) slab of an operand tile.
__device__ __forceinline__ void load_box(void* dst, const CUtensorMap* map, int mn_major, int mn0, int k0,
                                         int mat, uint64_t* bar) {
  if (mn_major)
    tma_load_3d(dst, map, bar, mn0, k0, mat);
  else
    tma_load_3d(dst, map, bar, k0, mn0, mat);
}

__device__ __forceinline__ uint64_t operand_desc(uint32_t tile_addr, int mn_major, int kk) {
  return mn_major ? smem_desc_sw128(tile_addr + kk * 2048u, 8192u, 1024u)
                  : smem_desc_sw128(tile_addr + kk * 32u, 16u, 1024u);
}

// ------------------------------------------------------------------ epilogue helpers

__device__ __forceinline__ void load_bf16x32(const __nv_bfloat16* src, float (&f)[32]) {
  const uint4* s4 = reinterpret_cast<const uint4*>(src);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint4 w = s4[q];
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      f[q * 8 + e * 2] = bf16_bits_to_float(ws[e] & 0xFFFFu);
      f[q * 8 + e * 2 + 1] = bf16_bits_to_float(ws[e] >> 16);
    }
  }
}

__device__ __forceinline__ void store_bf16x32(__nv_bfloat16* dst, const uint32_t (&bits)[32]) {
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    d4[q] = make_uint4(bits[q * 8 + 0] | (bits[q * 8 + 1] << 16), bits[q * 8 + 2] | (bits[q * 8 + 3] << 16),
                       bits[q * 8 + 4] | (bits[q * 8 + 5] << 16), bits[q * 8 + 6] | (bits[q * 8 + 7] << 16));
  }
}

__device__ __forceinline__ float bf16_at(const __nv_bfloat16* p) {
  return bf16_bits_to_float(__bfloat16_as_ushort(*p));
}

__device__ __forceinline__ void put_bf16(__nv_bfloat16* p, uint32_t bits) {
  *p = __ushort_as_bfloat16(static_cast<unsigned short>(bits));
}

// Symmetric products: thread owns tile row r; stores (R, C) for R <= C and mirrors it.
template <int MODE, int BN>
__device__ __forceinline__ void epilogue_sym(const GemmParams& p, const ClassDesc& cd, const Tile& tl, int r,
                                             uint32_t tacc) {
  const int m = cd.m;
  const int64_t lda = cd.lda;
  __nv_bfloat16* out = (MODE == kGram ? cd.a_buf : cd.b_buf) + tl.mat * cd.a_stride;
  const __nv_bfloat16* ain = cd.a_buf + tl.mat * cd.a_stride;
  const int R = tl.ib * kBM + r;
  float mul = 1.f;
  if (MODE == kGram && p.first_iter) {
    const float s = p.scale[cd.mat_base + tl.mat];
    mul = s * s;
  }
#pragma unroll 1
  for (int ch = 0; ch < BN / 32; ++ch) {
    const int C0 = tl.jb * BN + ch * 32;
    if (C0 >= m) break;  // uniform over the CTA
    float f[32];
    if (MODE == kPoly) {
      if (R < m) {
        if (C0 + 32 <= m) {
          load_bf16x32(ain + R * lda + C0, f);
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j) f[j] = (C0 + j < m) ? bf16_at(ain + R * lda + C0 + j) : 0.f;
        }
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) f[j] = 0.f;
      }
    }
    uint32_t v[32];
    tmem_ld_32x32b_x32(tacc + ch * 32, v);
    tmem_wait_ld();
    uint32_t bits[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const float acc = __uint_as_float(v[j]);
      const float val = (MODE == kPoly) ? fmaf(p.c, acc, p.b * f[j]) : acc * mul;
      bits[j] = float_to_bf16_bits(val);
    }
    if (R < m) {
      if (C0 >= R && C0 + 32 <= m) {
        store_bf16x32(out + R * lda + C0, bits);
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int C = C0 + j;
          if (C < m && C >= R) put_bf16(out + R * lda + C, bits[j]);
        }
      }
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const int C = C0 + j;
        if (C < m && C > R) put_bf16(out + static_cast<int64_t>(C) * lda + R, bits[j]);
      }
    }
  }
}

// X update: x_new = s (a (hi + lo) + acc); thread owns stored row R of the tile.
template <int MODE, int BN>
__device__ __forceinline__ void epilogue_apply(const typename ParamsOf<MODE>::type& p, const ClassDesc& cd,
                                               const Tile& tl, int r, uint32_t tacc) {
  const int rows = cd.rows, cols = cd.cols;
  const int R = tl.ib * kBM + r;
  const bool live = R < rows;
  const int64_t rowoff = tl.mat * cd.x_stride + static_cast<int64_t>(R) * cd.ldx;
  const __nv_bfloat16* hi_cur = cd.x_hi_cur + rowoff;
  __nv_bfloat16* hi_next = cd.x_hi_next + rowoff;
  __nv_bfloat16* lo = cd.x_lo + rowoff;
  const float s = p.first_iter ? p.scale[cd.mat_base + tl.mat] : 1.f;
  const float a = p.a;
#pragma unroll 1
  for (int ch = 0; ch < BN / 32; ++ch) {
    const int C0 = tl.jb * BN + ch * 32;
    if (C0 >= cols) break;  // uniform over the CTA
    const bool full = C0 + 32 <= cols;
    float xh[32], xl[32];
    if (live) {
      if (full) {
        load_bf16x32(hi_cur + C0, xh);
        load_bf16x32(lo + C0, xl);
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          xh[j] = (C0 + j < cols) ? bf16_at(hi_cur + C0 + j) : 0.f;
          xl[j] = (C0 + j < cols) ? bf16_at(lo + C0 + j) : 0.f;
        }
      }
    }
    uint32_t v[32];
    tmem_ld_32x32b_x32(tacc + ch * 32, v);
    tmem_wait_ld();
    if (!live) continue;
    float x[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) x[j] = s * fmaf(a, xh[j] + xl[j], __uint_as_float(v[j]));
    if constexpr (MODE == kApply) {
      uint32_t hb[32], lb[32];
#pragma unroll
      for (int j = 0; j < 32; ++j) split_hi_lo(x[j], hb[j], lb[j]);
      if (full) {
        store_bf16x32(hi_next + C0, hb);
        store_bf16x32(lo + C0, lb);
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          if (C0 + j < cols) {
            put_bf16(hi_next + C0 + j, hb[j]);
            put_bf16(lo + C0 + j, lb[j]);
          }
        }
      }
    } else {
      const UpdMat& u = p.upd[cd.mat_base + tl.mat];
      if (u.out != nullptr) {
        float* o = u.out + static_cast<int64_t>(R) * cols + C0;
        if (full && u.vec_out) {
#pragma unroll
          for (int q = 0; q < 8; ++q)
            reinterpret_cast<float4*>(o)[q] = make_float4(x[4 * q], x[4 * q + 1], x[4 * q + 2], x[4 * q + 3]);
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (C0 + j < cols) o[j] = x[j];
        }
      }
      if (u.param != nullptr) {
        const float decay = p.decay, ls = u.lr_scale;
        if (u.param_bf16) {
          __nv_bfloat16* w = static_cast<__nv_bfloat16*>(u.param) + static_cast<int64_t>(R) * u.ld_param + C0;
          if (full && u.vec_param) {
            float wf[32];
            load_bf16x32(w, wf);
            uint32_t wb[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) wb[j] = float_to_bf16_bits(fmaf(-ls, x[j], wf[j] * decay));
            store_bf16x32(w, wb);
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (C0 + j < cols) put_bf16(w + j, float_to_bf16_bits(fmaf(-ls, x[j], bf16_at(w + j) * decay)));
          }
        } else {
          float* w = static_cast<float*>(u.param) + static_cast<int64_t>(R) * u.ld_param + C0;
          if (full && u.vec_param) {
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              float4 t = reinterpret_cast<float4*>(w)[q];
              t.x = fmaf(-ls, x[4 * q], t.x * decay);
              t.y = fmaf(-ls, x[4 * q + 1], t.y * decay);
              t.z = fmaf(-ls, x[4 * q + 2], t.z * decay);
              t.w = fmaf(-ls, x[4 * q + 3], t.w * decay);
              reinterpret_cast<float4*>(w)[q] = t;
            }
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (C0 + j < cols) w[j] = fmaf(-ls, x[j], w[j] * decay);
          }
        }
      }
    }
  }
}

// ------------------------------------------------------------------ the kernel

template <int MODE, int BN>
__global__ void __launch_bounds__(kGemmThreads, 1)
    muon_ns_gemm_kernel(const __grid_constant__ typename ParamsOf<MODE>::type p) {
  using Cfg = GemmCfg<BN>;
  constexpr int S = Cfg::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S * Cfg::kStageBytes);
  uint64_t* empty = full + S;
  uint64_t* tfull = empty + S;
  uint64_t* tempty = tfull + 2;
  uint64_t* tdown = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tdown + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 4);
    }
    mbar_init(tdown, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    for (int c = 0; c < p.num_classes; ++c) {
      tma_prefetch_desc(&p.map_a[c]);
      tma_prefetch_desc(&p.map_b[c]);
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, Cfg::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const Watchdog wd{abort_flag, p.status, p.timeout_ns};

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      uint32_t armed = 0, armed_par = 0;  // stages with a load in flight, and its phase
      bool ok = true;
      for (int t = blockIdx.x; ok && t < p.total_tiles; t += gridDim.x) {
        const Tile tl = decode_tile<MODE, BN>(p, t);
        const ClassDesc& cd = p.cls[tl.cls];
        const CUtensorMap* ma = &p.map_a[tl.cls];
        const CUtensorMap* mb = &p.map_b[tl.cls];
        const int nk = (cd.ksize + kBK - 1) / kBK;
        const int a0 = tl.ib * kBM, b0 = tl.jb * BN;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&empty[s], ph ^ 1u, wd, kSiteProducerEmpty)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + s * Cfg::kStageBytes;
          uint8_t* sb = sa + Cfg::kABytes;
          mbar_arrive_expect_tx(&full[s], Cfg::kStageBytes);
          const int k0 = kb * kBK;
#pragma unroll
          for (int b = 0; b < kBM / kBox; ++b) load_box(sa + b * kBoxBytes, ma, cd.a_mn, a0 + b * kBox, k0, tl.mat, &full[s]);
#pragma unroll
          for (int b = 0; b < BN / kBox; ++b) load_box(sb + b * kBoxBytes, mb, cd.b_mn, b0 + b * kBox, k0, tl.mat, &full[s]);
          armed |= 1u << s;
          armed_par = (armed_par & ~(1u << s)) | (ph << s);
          if (++s == S) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
      if (!ok) {
        // Do not leave while a load may still write into this CTA's shared memory.
        const Watchdog quiet{abort_flag, p.status, teardown_budget(p.timeout_ns)};
        for (int k = 0; k < S; ++k) {
          if (armed & (1u << k)) {
            const uint32_t par = (armed_par >> k) & 1u;
            if (!mbar_try_wait(&full[k], par)) {
              const uint64_t t0 = global_timer_ns();
              while (!mbar_try_wait(&full[k], par) && global_timer_ns() - t0 < quiet.budget) {
              }
            }
          }
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      int s = 0, acc = 0;
      uint32_t ph = 0, aph = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < p.total_tiles; t += gridDim.x) {
        const Tile tl = decode_tile<MODE, BN>(p, t);
        const ClassDesc& cd = p.cls[tl.cls];
        const int nk = (cd.ksize + kBK - 1) / kBK;
        const uint32_t idesc = idesc_bf16_f32(kBM, BN, cd.a_mn, cd.b_mn);
        if (!mbar_wait(&tempty[acc], aph ^ 1u, wd, kSiteMmaTmemEmpty)) break;
        tc_fence_after();
        const uint32_t dtm = tmem_base + static_cast<uint32_t>(acc * BN);
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&full[s], ph, wd, kSiteMmaFull)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + s * Cfg::kStageBytes);
          const uint32_t sb = sa + Cfg::kABytes;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            umma_bf16(dtm, operand_desc(sa, cd.a_mn, kk), operand_desc(sb, cd.b_mn, kk), idesc,
                      (kb | kk) != 0 ? 1u : 0u);
          }
          umma_commit(&empty[s]);
          if (++s == S) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(&tfull[acc]);
        if (++acc == 2) {
          acc = 0;
          aph ^= 1u;
        }
      }
      // Every MMA this thread issued has finished before TMEM is released.
      umma_commit(tdown);
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(tdown, 0) && global_timer_ns() - t0 < teardown_budget(p.timeout_ns)) {
      }
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    const int q = warp & 3;  // TMEM lanes 32q..32q+31 are this warp's
    const int r = q * 32 + lane;
    int acc = 0;
    uint32_t aph = 0;
    for (int t = blockIdx.x; t < p.total_tiles; t += gridDim.x) {
      const Tile tl = decode_tile<MODE, BN>(p, t);
      const ClassDesc& cd = p.cls[tl.cls];
      int got = 0;
      if (lane == 0) got = mbar_wait(&tfull[acc], aph, wd, kSiteEpilogueFull) ? 1 : 0;
      got = __shfl_sync(0xffffffffu, got, 0);
      if (!got) break;
      tc_fence_after();
      const uint32_t tacc = tmem_base + static_cast<uint32_t>(acc * BN) + (static_cast<uint32_t>(q * 32) << 16);
      if constexpr (MODE == kGram || MODE == kPoly)
        epilogue_sym<MODE, BN>(p, cd, tl, r, tacc);
      else
        epilogue_apply<MODE, BN>(p, cd, tl, r, tacc);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
      if (++acc == 2) {
        acc = 0;
        aph ^= 1u;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, Cfg::kTmemCols);
  }
}

template <int MODE, int BN>
static cudaError_t launch_one(const typename ParamsOf<MODE>::type& p, int grid, cudaStream_t stream) {
  using Cfg = GemmCfg<BN>;
  static thread_local int configured_device = -1;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (configured_device != dev) {
    e = cudaFuncSetAttribute(muon_ns_gemm_kernel<MODE, BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             Cfg::kSmemBytes);
    if (e != cudaSuccess) return e;
    configured_device = dev;
  }
  muon_ns_gemm_kernel<MODE, BN><<<grid, kGemmThreads, Cfg::kSmemBytes, stream>>>(p);
  return cudaGetLastError();
}

int gemm_bn_for_mode(int mode) { return mode == kGram || mode == kPoly ? 128 : 256; }

cudaError_t launch_gemm(int mode, const GemmParams* p, int grid, cudaStream_t stream) {
  switch (mode) {
    case kGram: return launch_one<kGram, 128>(*p, grid, stream);
    case kPoly: return launch_one<kPoly, 128>(*p, grid, stream);
    case kApply: return launch_one<kApply, 256>(*p, grid, stream);
    case kApplyLast: return launch_one<kApplyLast, 256>(*static_cast<const FinalParams*>(p), grid, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace muon
