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
// CTA pairs.  The kernel runs as clusters of two CTAs on neighbouring SMs.  A pair
// computes a 256 x 256 output tile with tcgen05.mma.cta_group::2 (M = 256, N = 256,
// K = 16): each CTA stages its own 128 rows of the A operand and its own 128 rows
// (half of N) of the B operand, one thread of the leader CTA issues the MMAs, and
// each CTA's TMEM accumulates its 128 x 256 half of the tile.  Per SM that is a
// 32 KB stage for 128 x 256 x 64 of work, half the bytes per flop of a one-CTA
// 128 x 128 tile.  Both CTAs' loads complete on the leader's mbarrier; the leader's
// commits arrive on both CTAs' barriers; the peer's epilogue releases the
// accumulator by arriving on the leader's barrier.  No load uses cluster multicast.
//
// The Gram and the polynomial are symmetric: only pair tiles on or above the block
// diagonal are computed.  Each CTA looks at its two 128 x 128 blocks: a block above
// the diagonal is stored twice by TMA, as itself at (i, j) and transposed at (j, i);
// a diagonal block keeps its upper triangle and mirrors it into the lower one; a
// block below the diagonal is dropped.  Every element has one writer, and the stored
// matrices are exactly symmetric.
//
// A tall matrix (rows > cols) is never transposed in memory.  With Y the stored
// matrix (X = Y^T) the same iteration reads  A = Y^T Y  (both operands MN-major)
// and  Y <- a Y + Y B  (B symmetric), so operand majorness is a per-class run-time
// property of the launch.
//
// Roles in each CTA (320 threads, one CTA per SM, persistent over a flat tile list):
//   warp 0      one thread: TMA loads of 64 x 64 bf16 boxes (128-byte swizzle) into a
//               ring of shared-memory stages
//   warp 1      allocates TMEM for the pair (two fp32 accumulators of 128 x 256); in
//               the leader CTA one thread issues the MMAs and commits
//   warps 2..9  epilogue: tcgen05.ld (TMEM lane = tile row; warps w and w + 4 share a
//               lane quarter and split the columns), fused coefficient math in fp32,
//               results staged in shared memory (128-byte swizzle) and written by TMA
//               stores, one 128 x 128 block at a time.
// The epilogue of tile t overlaps the main loop of tile t + 1.
#include "muon_device.cuh"
#include "muon_params.h"

#include <algorithm>

namespace muon {

template <int MODE>
struct Lay {
  static constexpr bool kSym = MODE == kGram || MODE == kPoly;
  static constexpr int TM = 256;  // pair tile rows (128 per CTA)
  static constexpr int TN = 256;  // pair tile columns = UMMA N
  static constexpr int S = MODE == kGram ? 5 : 3;
  static constexpr int NEPI = 8;
  static constexpr int kABytes = kBM * kBK * 2;  // this CTA's 128 rows of A
  static constexpr int kBBytes = kBM * kBK * 2;  // this CTA's 128 rows (half of N) of B
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kRing = S * kStageBytes;
  static constexpr int kBlk = kBM * 128 * 2;  // one staged 128 x 128 bf16 block
  // Gram: D, T.  Polynomial: D, T, Ain (128 x 256).  Apply: hi, lo (128 x 256 each).
  static constexpr int kEpi = MODE == kGram ? 2 * kBlk : 4 * kBlk;
  static constexpr int kBarOff = kRing + kEpi;
  static constexpr int kSmemBytes = kBarOff + 256 + 1024;
  static constexpr int kEpiThreads = 32 * NEPI;
  static constexpr int kThreads = 64 + kEpiThreads;
  static constexpr int kTmemCols = 2 * TN;
  static_assert(kSmemBytes <= 232448, "shared memory budget");
};

template <int MODE>
struct ParamsOf {
  using type = GemmParams;
};
template <>
struct ParamsOf<kApplyLast> {
  using type = FinalParams;
};

// Waits on the way out (loads and MMAs already in flight) get at least two seconds,
// whatever the per-wait budget: they end by themselves, and leaving before they do
// would let a copy land in shared memory this CTA no longer owns.
__device__ __forceinline__ unsigned long long teardown_budget(unsigned long long budget) {
  return budget > 2000000000ull ? budget : 2000000000ull;
}

__device__ __forceinline__ void quiet_wait(uint64_t* bar, uint32_t parity, unsigned long long budget) {
  if (mbar_try_wait(bar, parity)) return;
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity) && global_timer_ns() - t0 < budget) {
  }
}

// Lane 0 waits, the warp learns the outcome (keeps .sync.aligned tcgen05 ops convergent).
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, const Watchdog& w, int site) {
  int ok = 0;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, w, site) ? 1 : 0;
  return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

// A pair tile: class, matrix within the class, 256-row block I, 256-column block J.
struct Tile {
  int cls, mat, I, J;
};

template <int MODE>
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
    // upper block triangle, row by row: row I holds column blocks I .. nb-1
    int I = 0;
    while (q >= cd.nb - I) {
      q -= cd.nb - I;
      ++I;
    }
    r.I = I;
    r.J = I + q;
  } else if (cd.i_fast) {
    r.I = q % cd.mb;
    r.J = q / cd.mb;
  } else {
    r.J = q % cd.nb;
    r.I = q / cd.nb;
  }
  return r;
}

// One 64-row (K-major) or 64-column (MN-major) slab of an operand tile, completing on
// the leader CTA's mbarrier.
__device__ __forceinline__ void load_box_pair(void* dst, const CUtensorMap* map, int mn_major, int mn0, int k0,
                                              int mat, uint32_t bar_cluster) {
  if (mn_major)
    tma_load_3d_pair(dst, map, bar_cluster, mn0, k0, mat);
  else
    tma_load_3d_pair(dst, map, bar_cluster, k0, mn0, mat);
}

__device__ __forceinline__ uint64_t operand_desc(uint32_t tile_addr, int mn_major, int kk) {
  return mn_major ? smem_desc_sw128(tile_addr + kk * 2048u, 8192u, 1024u)
                  : smem_desc_sw128(tile_addr + kk * 32u, 16u, 1024u);
}

// ------------------------------------------------------------------ staging layouts
//
// A staged region of 128 rows x (64 NCB) columns of bf16 is a grid of 64 x 64 boxes with
// 128-byte swizzle, as TMA reads and writes them: box (rb, cb) at (rb NCB + cb) * 8 KB,
// row rr of a box at rr * 128 B, and its 16-byte chunk k at chunk k ^ (rr & 7).  Eight
// consecutive rows then hit eight different bank groups: conflict-free row access.
template <int NCB>
__device__ __forceinline__ uint32_t chunk_off(int r, int c16) {
  const int rr = r & 63;
  return static_cast<uint32_t>((((r >> 6) * NCB + (c16 >> 3)) << 13) + rr * 128 + (((c16 & 7) ^ (rr & 7)) << 4));
}

template <int NCB>
__device__ __forceinline__ uint32_t elem_off(int r, int c) {
  return chunk_off<NCB>(r, c >> 3) + ((c & 7) << 1);
}

__device__ __forceinline__ void unpack8(uint4 w, float* f) {
  const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    f[2 * e] = bf16_bits_to_float(ws[e] & 0xFFFFu);
    f[2 * e + 1] = bf16_bits_to_float(ws[e] >> 16);
  }
}

__device__ __forceinline__ uint4 pack8(const uint32_t* b) {
  return make_uint4(b[0] | (b[1] << 16), b[2] | (b[3] << 16), b[4] | (b[5] << 16), b[6] | (b[7] << 16));
}

__device__ __forceinline__ void st_u16(uint8_t* base, uint32_t off, uint32_t bits) {
  *reinterpret_cast<unsigned short*>(base + off) = static_cast<unsigned short>(bits);
}

__device__ __forceinline__ float bf16_at(const __nv_bfloat16* p) {
  return bf16_bits_to_float(__bfloat16_as_ushort(*p));
}

__device__ __forceinline__ void put_bf16(__nv_bfloat16* p, uint32_t bits) {
  *p = __ushort_as_bfloat16(static_cast<unsigned short>(bits));
}

// Stores / loads a staged region of 128 rows x 64 NCB columns at rows row0.., columns
// col0.. of matrix `mat`; parts outside the matrix are not written / read as zero.
template <int NCB>
__device__ __forceinline__ void store_region(const CUtensorMap* map, const uint8_t* buf, int cb0, int ncb, int row0,
                                             int col0, int mat) {
#pragma unroll 1
  for (int rb = 0; rb < 2; ++rb)
#pragma unroll 1
    for (int cb = cb0; cb < cb0 + ncb; ++cb)
      tma_store_3d(map, buf + ((rb * NCB + cb) << 13), col0 + 64 * cb, row0 + 64 * rb, mat);
}

template <int NCB>
__device__ __forceinline__ void load_region(uint8_t* buf, const CUtensorMap* map, uint64_t* bar, int row0, int col0,
                                            int mat) {
#pragma unroll
  for (int rb = 0; rb < 2; ++rb)
#pragma unroll
    for (int cb = 0; cb < NCB; ++cb)
      tma_load_3d(buf + ((rb * NCB + cb) << 13), map, bar, col0 + 64 * cb, row0 + 64 * rb, mat);
}

// ------------------------------------------------------------------ epilogues

// One 128 x 128 block of a symmetric product: block row r of this CTA, the 64 columns
// [64 h, 64 h + 64) of the block; the block's accumulator columns start at 128 hh.
// Off-diagonal: the row goes to D, its transpose to T.  Diagonal: D gets the upper
// triangle from the row owners and the lower triangle mirrored from it.
template <int MODE>
__device__ __forceinline__ void sym_block(const GemmParams& p, float mul, bool diag, int r, int h, int hh,
                                          uint32_t tacc, uint8_t* D, uint8_t* T, const uint8_t* Ain) {
#pragma unroll 1
  for (int k = 0; k < 2; ++k) {
    const int c0 = 64 * h + 32 * k;
    uint32_t v[32];
    tmem_ld_32x32b_x32(tacc + 128 * hh + c0, v);
    float f[32];
    if (MODE == kPoly) {
#pragma unroll
      for (int q = 0; q < 4; ++q)
        unpack8(*reinterpret_cast<const uint4*>(Ain + chunk_off<4>(r, ((128 * hh + c0) >> 3) + q)), f + 8 * q);
    }
    tmem_wait_ld();
    uint32_t bits[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const float acc = __uint_as_float(v[j]);
      bits[j] = float_to_bf16_bits(MODE == kPoly ? fmaf(p.c, acc, p.b * f[j]) : acc * mul);
    }
    if (!diag) {
#pragma unroll
      for (int q = 0; q < 4; ++q)
        *reinterpret_cast<uint4*>(D + chunk_off<2>(r, (c0 >> 3) + q)) = pack8(bits + 8 * q);
#pragma unroll
      for (int j = 0; j < 32; ++j) st_u16(T, elem_off<2>(c0 + j, r), bits[j]);
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const int c = c0 + j;
        if (c >= r) st_u16(D, elem_off<2>(r, c), bits[j]);
        if (c > r) st_u16(D, elem_off<2>(c, r), bits[j]);
      }
    }
  }
}

// X update for the 32 tile columns [c0, c0 + 32) of this CTA's tile row r:
// x = s (a (hi + lo) + acc), hi/lo read from the staged 128 x 256 input region.  kApply
// writes the new hi/lo pair back in place; kApplyLast updates W and/or writes O.
template <int MODE>
__device__ __forceinline__ void apply_cols(const typename ParamsOf<MODE>::type& p, const ClassDesc& cd,
                                           const Tile& tl, int rank, int r, int c0, uint32_t tacc, uint8_t* hib,
                                           uint8_t* lob, float s) {
  uint32_t v[32];
  tmem_ld_32x32b_x32(tacc + c0, v);
  float xh[32], xl[32];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const uint32_t o = chunk_off<4>(r, (c0 >> 3) + q);
    unpack8(*reinterpret_cast<const uint4*>(hib + o), xh + 8 * q);
    unpack8(*reinterpret_cast<const uint4*>(lob + o), xl + 8 * q);
  }
  tmem_wait_ld();
  float x[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) x[j] = s * fmaf(p.a, xh[j] + xl[j], __uint_as_float(v[j]));
  if constexpr (MODE == kApply) {
    uint32_t hb[32], lb[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) split_hi_lo(x[j], hb[j], lb[j]);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t o = chunk_off<4>(r, (c0 >> 3) + q);
      *reinterpret_cast<uint4*>(hib + o) = pack8(hb + 8 * q);
      *reinterpret_cast<uint4*>(lob + o) = pack8(lb + 8 * q);
    }
  } else {
    const int R = Lay<MODE>::TM * tl.I + kBM * rank + r;
    const int C0 = Lay<MODE>::TN * tl.J + c0;
    const int cols = cd.cols;
    if (R >= cd.rows || C0 >= cols) return;
    const bool full = C0 + 32 <= cols;
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
          uint4 raw[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) raw[q] = reinterpret_cast<const uint4*>(w)[q];
          uint32_t wb[32];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            float wf[8];
            unpack8(raw[q], wf);
#pragma unroll
            for (int e = 0; e < 8; ++e) wb[8 * q + e] = float_to_bf16_bits(fmaf(-ls, x[8 * q + e], wf[e] * decay));
          }
#pragma unroll
          for (int q = 0; q < 4; ++q) reinterpret_cast<uint4*>(w)[q] = pack8(wb + 8 * q);
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

// ------------------------------------------------------------------ the kernel

template <int MODE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(Lay<MODE>::kThreads, 1)
    muon_ns_gemm_kernel(const __grid_constant__ typename ParamsOf<MODE>::type p) {
  using L = Lay<MODE>;
  constexpr int S = L::S;
  constexpr bool kSym = L::kSym;
  constexpr int NT = L::kEpiThreads;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* epi = smem + L::kRing;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBarOff);  // used in the leader CTA
  uint64_t* empty = full + S;
  uint64_t* tfull = empty + S;
  uint64_t* tempty = tfull + 2;  // used in the leader CTA: both CTAs' epilogues arrive
  uint64_t* tdown = tempty + 2;
  uint64_t* efull = tdown + 1;  // this CTA's epilogue inputs landed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(efull + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* epi_flag = abort_flag + 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int rank = static_cast<int>(cluster_rank());
  const bool leader_cta = rank == 0;
  const int pair = blockIdx.x >> 1;
  const int npairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 2 * L::NEPI);
    }
    mbar_init(tdown, 1);
    mbar_init(efull, 1);
    *abort_flag = 0;
    *epi_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    for (int c = 0; c < p.num_classes; ++c) {
      tma_prefetch_desc(&p.map_a[c]);
      tma_prefetch_desc(&p.map_b[c]);
    }
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, L::kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the peer's barriers exist before anything arrives on them
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const Watchdog wd{abort_flag, p.status, p.timeout_ns};
  const unsigned long long tb = teardown_budget(p.timeout_ns);

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer (both CTAs)
    if (lane == 0) {
      const uint32_t full0 = map_to_rank(smem_u32(full), 0);
      int s = 0;
      uint32_t ph = 0;
      uint32_t armed = 0, armed_par = 0;
      bool ok = true;
      for (int t = pair; ok && t < p.total_tiles; t += npairs) {
        const Tile tl = decode_tile<MODE>(p, t);
        const ClassDesc& cd = p.cls[tl.cls];
        const int row0 = L::TM * tl.I + kBM * rank;
        const CUtensorMap* ma = &p.map_a[tl.cls];
        const CUtensorMap* mb = &p.map_b[tl.cls];
        const int nk = (cd.ksize + kBK - 1) / kBK;
        const int b0 = L::TN * tl.J + kBM * rank;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&empty[s], ph ^ 1u, wd, kSiteProducerEmpty)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + s * L::kStageBytes;
          uint8_t* sb = sa + L::kABytes;
          if (leader_cta) mbar_arrive_expect_tx(&full[s], 2 * L::kStageBytes);
          const uint32_t fb = full0 + 8u * static_cast<uint32_t>(s);
          const int k0 = kb * kBK;
#pragma unroll
          for (int b = 0; b < kBM / kBox; ++b) load_box_pair(sa + b * kBoxBytes, ma, cd.a_mn, row0 + b * kBox, k0, tl.mat, fb);
#pragma unroll
          for (int b = 0; b < kBM / kBox; ++b) load_box_pair(sb + b * kBoxBytes, mb, cd.b_mn, b0 + b * kBox, k0, tl.mat, fb);
          armed |= 1u << s;
          armed_par = (armed_par & ~(1u << s)) | (ph << s);
          if (++s == S) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
      if (!ok) {
        // Do not leave while a load may still write into shared memory.  The peer's
        // operand bytes complete on the leader's barriers, which the leader waits for
        // here; the final cluster barrier keeps the peer until then.
        if (leader_cta)
          for (int j = 0; j < S; ++j)
            if (armed & (1u << j)) quiet_wait(&full[j], (armed_par >> j) & 1u, tb);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer (leader CTA)
    if (lane == 0) {
      if (leader_cta) {
        int s = 0, acc = 0;
        uint32_t ph = 0, aph = 0;
        bool ok = true;
        for (int t = pair; ok && t < p.total_tiles; t += npairs) {
          const Tile tl = decode_tile<MODE>(p, t);
          const ClassDesc& cd = p.cls[tl.cls];
          const int nk = (cd.ksize + kBK - 1) / kBK;
          const uint32_t idesc = idesc_bf16_f32(L::TM, L::TN, cd.a_mn, cd.b_mn);
          if (!mbar_wait(&tempty[acc], aph ^ 1u, wd, kSiteMmaTmemEmpty)) break;
          tc_fence_after();
          const uint32_t dtm = tmem_base + static_cast<uint32_t>(acc * L::TN);
          for (int kb = 0; kb < nk; ++kb) {
            if (!mbar_wait(&full[s], ph, wd, kSiteMmaFull)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t sa = smem_u32(smem + s * L::kStageBytes);
            const uint32_t sb = sa + L::kABytes;
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk)
              umma_bf16_pair(dtm, operand_desc(sa, cd.a_mn, kk), operand_desc(sb, cd.b_mn, kk), idesc,
                             (kb | kk) != 0 ? 1u : 0u);
            umma_commit_pair(&empty[s], 0x3);
            if (++s == S) {
              s = 0;
              ph ^= 1u;
            }
          }
          if (!ok) break;
          umma_commit_pair(&tfull[acc], 0x3);
          if (++acc == 2) {
            acc = 0;
            aph ^= 1u;
          }
        }
        // Every MMA has finished (in both CTAs' TMEM and shared memory) before either
        // CTA releases TMEM or leaves.
        umma_commit_pair(tdown, 0x3);
      }
      quiet_wait(tdown, 0, tb);
    }
  } else {
    // ---------------------------------------------------------------- epilogue (both CTAs)
    const int ew = warp - 2;
    const int q = warp & 3;  // TMEM lanes 32q..32q+31 belong to this warp
    const int h = ew >> 2;   // column group within a 128-column block
    const int r = q * 32 + lane;
    const bool leader = threadIdx.x == 64;
    const uint32_t tempty0 = map_to_rank(smem_u32(tempty), 0);
    uint8_t* D = epi;
    uint8_t* T = epi + L::kBlk;
    uint8_t* Ain = epi + 2 * L::kBlk;
    int acc = 0;
    uint32_t aph = 0;
    // Epilogue inputs (polynomial: A; apply: hi and lo) for tile t are loaded by the
    // epilogue leader as soon as tile t - 1 no longer needs the buffer, so the main
    // loop never waits on them.
    bool in_pending = false;
    uint32_t in_par = 0;
    auto load_inputs = [&](int tt) {
      const Tile nx = decode_tile<MODE>(p, tt);
      const int row0 = L::TM * nx.I + kBM * rank, col0 = L::TN * nx.J;
      fence_proxy_async_smem();
      if constexpr (MODE == kPoly) {
        mbar_arrive_expect_tx(efull, 2 * L::kBlk);
        load_region<4>(Ain, &p.map_in0[nx.cls], efull, row0, col0, nx.mat);
      } else {
        mbar_arrive_expect_tx(efull, 4 * L::kBlk);
        load_region<4>(epi, &p.map_in0[nx.cls], efull, row0, col0, nx.mat);
        load_region<4>(epi + 2 * L::kBlk, &p.map_in1[nx.cls], efull, row0, col0, nx.mat);
      }
      in_pending = true;
    };
    if (MODE != kGram && leader && pair < p.total_tiles) load_inputs(pair);
    int k = 0;
    for (int t = pair; t < p.total_tiles; t += npairs, ++k) {
      const Tile tl = decode_tile<MODE>(p, t);
      const ClassDesc& cd = p.cls[tl.cls];
      const uint32_t kpar = static_cast<uint32_t>(k) & 1u;
      // One warp waits for the accumulator (and the staged inputs); the rest learn the
      // outcome at the barrier, so every epilogue warp leaves the loop together.
      if (ew == 0) {
        bool ok = warp_wait(&tfull[acc], aph, wd, kSiteEpilogueFull);
        if (ok && MODE != kGram) ok = warp_wait(efull, kpar, wd, kSiteEpilogueIn);
        if (lane == 0) *epi_flag = ok ? 1 : 0;
      }
      named_barrier(1, NT);
      if (*epi_flag == 0) break;
      if (MODE != kGram) {
        in_pending = false;
        in_par = kpar ^ 1u;
      }
      tc_fence_after();
      const uint32_t tacc = tmem_base + static_cast<uint32_t>(acc * L::TN) + (static_cast<uint32_t>(q * 32) << 16);
      if constexpr (kSym) {
        const int rb = 2 * tl.I + rank;  // this CTA's 128-row block
        float mul = 1.f;
        if (MODE == kGram && p.first_iter) {
          const float sv = p.scale[cd.mat_base + tl.mat];
          mul = sv * sv;
        }
        bool stored = false;
#pragma unroll 1
        for (int hh = 0; hh < 2; ++hh) {
          const int cb = 2 * tl.J + hh;
          if (rb > cb) continue;  // below the diagonal: its mirror is stored by another block
          if (stored) {
            if (leader) bulk_wait_read<0>();
            named_barrier(1, NT);  // D and T free again
          }
          sym_block<MODE>(p, mul, rb == cb, r, h, hh, tacc, D, T, Ain);
          fence_proxy_async_smem();
          named_barrier(1, NT);
          if (leader) {
            const CUtensorMap* mo = &p.map_out[tl.cls];
            store_region<2>(mo, D, 0, 2, kBM * rb, kBM * cb, tl.mat);
            if (rb < cb) store_region<2>(mo, T, 0, 2, kBM * cb, kBM * rb, tl.mat);
            bulk_commit();
          }
          stored = true;
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(tempty0 + 8u * static_cast<uint32_t>(acc));
        if (leader) {
          if (MODE == kPoly && t + npairs < p.total_tiles) load_inputs(t + npairs);
          bulk_wait_read<0>();  // D and T are free for the next tile
        }
      } else {
        uint8_t* hib = epi;
        uint8_t* lob = epi + 2 * L::kBlk;
        const float sc = p.first_iter ? p.scale[cd.mat_base + tl.mat] : 1.f;
#pragma unroll 1
        for (int hh = 0; hh < 2; ++hh) {
          apply_cols<MODE>(p, cd, tl, rank, r, 128 * hh + 64 * h, tacc, hib, lob, sc);
          apply_cols<MODE>(p, cd, tl, rank, r, 128 * hh + 64 * h + 32, tacc, hib, lob, sc);
          if (hh == 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(tempty0 + 8u * static_cast<uint32_t>(acc));
          }
          if constexpr (MODE == kApply) {
            fence_proxy_async_smem();
            named_barrier(1, NT);
            if (leader) {
              const int row0 = L::TM * tl.I + kBM * rank, col0 = L::TN * tl.J;
              store_region<4>(&p.map_out[tl.cls], hib, 2 * hh, 2, row0, col0, tl.mat);
              store_region<4>(&p.map_in1[tl.cls], lob, 2 * hh, 2, row0, col0, tl.mat);
              bulk_commit();
            }
          }
        }
        if constexpr (MODE == kApply) {
          if (leader) {
            bulk_wait_read<0>();  // the stores have read the region: it can be refilled
            if (t + npairs < p.total_tiles) load_inputs(t + npairs);
          }
        } else {
          named_barrier(1, NT);  // every thread is done reading the input region
          if (leader && t + npairs < p.total_tiles) load_inputs(t + npairs);
        }
      }
      if (++acc == 2) {
        acc = 0;
        aph ^= 1u;
      }
    }
    if (leader) {
      bulk_wait_all();
      if (in_pending) quiet_wait(efull, in_par, tb);
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // nothing arrives on, or lands in, either CTA after this point
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, L::kTmemCols);
  }
}

template <int MODE>
static cudaError_t launch_one(const typename ParamsOf<MODE>::type& p, int max_pairs, cudaStream_t stream) {
  using L = Lay<MODE>;
  static thread_local int configured_device = -1;
  static thread_local int resident_pairs = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (configured_device != dev) {
    e = cudaFuncSetAttribute(muon_ns_gemm_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kSmemBytes);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * max_pairs, 1, 1);
    cfg.blockDim = dim3(L::kThreads, 1, 1);
    cfg.dynamicSmemBytes = L::kSmemBytes;
    int clusters = 0;
    e = cudaOccupancyMaxActiveClusters(&clusters, muon_ns_gemm_kernel<MODE>, &cfg);
    if (e != cudaSuccess) return e;
    resident_pairs = clusters > 0 ? clusters : 1;
    configured_device = dev;
  }
  const int pairs = std::max(1, std::min(std::min(p.total_tiles, max_pairs), resident_pairs));
  muon_ns_gemm_kernel<MODE><<<2 * pairs, L::kThreads, L::kSmemBytes, stream>>>(p);
  return cudaGetLastError();
}

int gemm_tile_rows() { return 256; }
int gemm_tile_cols() { return 256; }

// `max_pairs` bounds the number of CTA pairs (half the SM count).
cudaError_t launch_gemm(int mode, const GemmParams* p, int max_pairs, cudaStream_t stream) {
  switch (mode) {
    case kGram: return launch_one<kGram>(*p, max_pairs, stream);
    case kPoly: return launch_one<kPoly>(*p, max_pairs, stream);
    case kApply: return launch_one<kApply>(*p, max_pairs, stream);
    case kApplyLast: return launch_one<kApplyLast>(*static_cast<const FinalParams*>(p), max_pairs, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace muon
