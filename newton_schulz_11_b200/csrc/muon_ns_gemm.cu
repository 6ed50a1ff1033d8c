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
// matrices are exactly symmetric.  On a diagonal pair tile each CTA's A rows are its B
// rows, so its stages hold one operand tile and the MMAs read it as both.
//
// A tall matrix (rows > cols) is never transposed in memory.  With Y the stored
// matrix (X = Y^T) the same iteration reads  A = Y^T Y  (both operands MN-major)
// and  Y <- a Y + Y B  (B symmetric), so operand majorness is a per-class run-time
// property of the launch.
//
// Roles in each CTA (320 threads, 352 in the staged applies; one CTA per SM, persistent
// over a flat tile list):
//   warp 0      one thread: TMA loads of 64 x 64 bf16 boxes (128-byte swizzle) into a
//               ring of shared-memory stages
//   warp 1      allocates TMEM for the pair (two fp32 accumulators of 128 x 256); in
//               the leader CTA one thread issues the MMAs and commits
//   warps 2..9  epilogue: tcgen05.ld (TMEM lane = tile row; warps w and w + 4 share a
//               lane quarter and split the columns), fused coefficient math in fp32,
//               results staged in shared memory (128-byte swizzle) and written by TMA
//               stores, one 128 x 128 block at a time (the staged applies write theirs
//               straight from registers instead)
//   warp 10     staged applies only: TMA loads of the epilogue's inputs (the tile's old hi
//               and lo), a 64-column quarter at a time, each as soon as every epilogue warp
//               has read the quarter it replaces
// The epilogue of tile t overlaps the main loop of tile t + 1.
#include "muon_device.cuh"
#include "muon_params.h"

#include <algorithm>

namespace muon {

// Two variants share the kernel.
//   Streamed (SMALL = false, for long reductions): 128-deep k-blocks, three 64 KB stages
//   per CTA, one 32 KB epilogue staging area; epilogue inputs are read from global memory.
//   Staged (SMALL = true, when every Gram side m of the launch is at most 1024): 64-deep
//   k-blocks in 32 KB stages, and the epilogue's inputs moved by TMA through shared
//   memory -- there tiles are short, and the epilogue, not the main loop, sets the pace.
//     Gram        five stages; two 32 KB output staging buffers (stores of one quarter
//                 drain while the next is written); not used (the Gram streams)
//     polynomial  four stages; one output buffer; the tile's A block (64 KB) staged
//     apply       five stages (the last apply four); the tile's old hi and 8-bit lo staged
//                 by the loader warp in 24 KB quarter slots, two (four); the new hi and lo
//                 (or W and O) written with 32-byte global stores, so no epilogue warp
//                 waits for a store or for another warp
template <int MODE, int VAR = kStreamed>
struct Lay {
  static constexpr bool kSym = MODE == kGram || MODE == kPoly;
  static constexpr bool SMALL = VAR == kStaged;
  static constexpr bool kLoader = SMALL && !kSym;  // staged applies: a warp stages the epilogue's inputs
  // staged applies: 64-column quarters of the tile's old hi (16 KB) and lo (8 KB) in flight.
  // The apply takes a fifth operand stage in place of two of the four slots (measured
  // faster); the last apply, whose epilogue also reads and writes W, keeps four of each
  // (five and two measured 2.5% slower there).
  static constexpr int kSlots = !kLoader ? 0 : MODE == kApply ? 2 : 4;
  static constexpr int kSlotBytes = 3 * kBM * 64;  // 24 KB
  static constexpr int TM = 256;  // pair tile rows (128 per CTA)
  static constexpr int TN = 256;  // pair tile columns = UMMA N
  static constexpr int BK = VAR == kStreamed ? 128 : 64;
  // staged symmetric products: output staging buffers (32 KB each).  The polynomial takes
  // one, and a fourth operand stage with the space (measured faster than two and three).
  static constexpr int kOutBufs = MODE == kPoly ? 1 : 2;
  static constexpr int S = !SMALL ? 3 : (MODE == kGram ? 5 : (kSym ? (kOutBufs == 1 ? 4 : 3) : (MODE == kApply ? 5 : 4)));
  // epilogue warps; in the staged applies each handles 256 / NEPI columns of every quarter
  // (16 warps, or the new hi/lo written back into the slot and stored by TMA from the
  // loader warp, measured slower there)
  static constexpr int NEPI = 8;
  static constexpr int kBox64 = 64 * 64 * 2;       // one 64 x 64 box: 8 KB
  static constexpr int kHalf = kBM * kBox * 2;      // one 64 x 128 box: 16 KB
  static constexpr int kABytes = kBM * BK * 2;      // this CTA's 128 rows x BK of A
  static constexpr int kBBytes = kBM * BK * 2;      // this CTA's 128 rows (half of N) x BK of B
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kRing = S * kStageBytes;
  // streamed: one 64-column quarter of this CTA's 128 x 256 tile at a time (symmetric
  // modes D_q and T_q, apply hi_q and lo_q); staged: see above
  static constexpr int kEpi = !SMALL ? 2 * kHalf
                                     : (MODE == kGram ? 4 * kHalf : (kSym ? (4 + 2 * kOutBufs) * kHalf : kSlots * kSlotBytes));
  static constexpr int kBarOff = kRing + kEpi;
  static constexpr int kSmemBytes = kBarOff + 256 + 1024;
  static constexpr int kEpiThreads = 32 * NEPI;
  static constexpr int kLoaderWarp = 2 + NEPI;
  static constexpr int kThreads = 64 + kEpiThreads + (kLoader ? 32 : 0);
  static constexpr int kTmemCols = 2 * TN;
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  static_assert(S <= 8, "barrier area");
  static_assert(TM == TN && kABytes == kBBytes, "diagonal tiles read one operand tile as both");
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

// A diagonal pair tile (I == J) of a symmetric product: each CTA's A rows are its B rows
// (both operands are the same matrix through the same tensor map, and TM == TN), so the
// stage holds one operand tile and the MMA reads it as both.
template <int MODE>
__device__ __forceinline__ bool is_diag_tile(const Tile& tl) {
  return (MODE == kGram || MODE == kPoly) && tl.I == tl.J;
}

// This CTA's bytes in stage-load i (issue order) of pair `pair`; used only to settle the
// loads left open after a timeout.
template <int MODE, class L>
__device__ uint32_t load_share_bytes(const GemmParams& p, int pair, int npairs, uint32_t i) {
  for (int t = pair; t < p.total_tiles; t += npairs) {
    const Tile tl = decode_tile<MODE>(p, t);
    const uint32_t nk = static_cast<uint32_t>((p.cls[tl.cls].ksize + L::BK - 1) / L::BK);
    if (i < nk) return is_diag_tile<MODE>(tl) ? L::kABytes : L::kStageBytes;
    i -= nk;
  }
  return L::kStageBytes;
}

// One operand tile (128 MN x BK) into `dst`, completing on the leader CTA's mbarrier.
//   BK = 128 (64 x 128 boxes): K-major -> two boxes, K columns [k0 + 64 i, +64) of 128 rows;
//                              MN-major -> two boxes, MN columns [mn0 + 64 i, +64) of 128 K-rows.
//   BK = 64: K-major (64 x 128 box) -> one box, 64 K columns of 128 rows;
//            MN-major (64 x 64 boxes) -> two boxes, MN columns [mn0 + 64 i, +64) of 64 K-rows.
// Box i lands at i x (its bytes), which is the layout operand_desc reads.
template <int BK>
__device__ __forceinline__ void load_operand_pair(uint8_t* dst, const CUtensorMap* map, int mn_major, int mn0, int k0,
                                                  int mat, uint32_t bar_cluster) {
  constexpr int kBoxBytes = kBM * BK;  // half of the tile's bytes
  if (mn_major) {
    tma_load_3d_pair(dst, map, bar_cluster, mn0, k0, mat);
    tma_load_3d_pair(dst + kBoxBytes, map, bar_cluster, mn0 + 64, k0, mat);
  } else if (BK == 128) {
    tma_load_3d_pair(dst, map, bar_cluster, k0, mn0, mat);
    tma_load_3d_pair(dst + kBoxBytes, map, bar_cluster, k0 + 64, mn0, mat);
  } else {
    tma_load_3d_pair(dst, map, bar_cluster, k0, mn0, mat);
  }
}

// Shared-memory descriptor of the kk-th 16-deep K slice (kk < BK / 16) of a staged operand:
//   K-major : 128 rows x 128 B per 64-deep K half (16 KB); slice kk in half kk / 4, 32 B per
//             slice; 8-row groups 1 KB apart (SBO).
//   MN-major: two halves (64 MN each) of BK K-rows x 128 B; slice kk starts at K-row 16 kk
//             (2 KB per slice); 8-row groups 1 KB apart (SBO), halves BK x 128 B apart (LBO).
template <int BK>
__device__ __forceinline__ uint64_t operand_desc(uint32_t tile_addr, int mn_major, int kk) {
  return mn_major ? smem_desc_sw128(tile_addr + kk * 2048u, BK * 128u, 1024u)
                  : smem_desc_sw128(tile_addr + (kk >> 2) * 16384u + (kk & 3) * 32u, 16u, 1024u);
}

// ------------------------------------------------------------------ staging layouts
//
// Epilogue staging, as TMA stores read it (64 x 64 boxes, 128-byte swizzle: row rr of a box at
// rr * 128 B, its 16-byte chunk k at chunk k ^ (rr & 7)):
//   Q (offset 0)     128 rows x 64 columns: D_q, or the new hi of the apply
//   T (offset 16 KB) symmetric modes: 64 rows x 128 columns (the transpose of D_q), as two
//                    boxes side by side; apply: 128 x 64, the new lo, laid out like Q
// Eight consecutive rows hit eight different bank groups: row-wise access is conflict-free.
__device__ __forceinline__ uint32_t q_chunk(int r, int c16) { return static_cast<uint32_t>(r * 128 + ((c16 ^ (r & 7)) << 4)); }

// Staged apply: the tile's hi (and lo) as 128 rows x 256 columns, a 2 x 4 grid of 64 x 64
// boxes in the same swizzle: box (rb, cb) at (4 rb + cb) x 8 KB.
__device__ __forceinline__ uint32_t region_chunk(int r, int c16) {
  const int rr = r & 63;
  return static_cast<uint32_t>((((r >> 6) * 4 + (c16 >> 3)) << 13) + rr * 128 + (((c16 & 7) ^ (rr & 7)) << 4));
}

// A staged 128-row x 64-column bf16 quarter, two 64 x 64 boxes (rows 0-63, then 64-127) in the
// same swizzle: row r's 16-byte chunk c (0..7).
__device__ __forceinline__ uint32_t quarter_chunk(int r, int c16) {
  const int rr = r & 63;
  return static_cast<uint32_t>(((r >> 6) << 13) + rr * 128 + ((c16 ^ (rr & 7)) << 4));
}

// Loads column box cb (both row boxes) of the staged region.
__device__ __forceinline__ void load_region_quarter(uint8_t* buf, const CUtensorMap* map, uint64_t* bar, int cb,
                                                    int row0, int col0, int mat) {
#pragma unroll
  for (int rb = 0; rb < 2; ++rb)
    tma_load_3d(buf + ((4 * rb + cb) << 13), map, bar, col0 + 64 * cb, row0 + 64 * rb, mat);
}

__device__ __forceinline__ uint4 pack8(const uint32_t* b) {
  return make_uint4(b[0] | (b[1] << 16), b[2] | (b[3] << 16), b[4] | (b[5] << 16), b[6] | (b[7] << 16));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

__device__ __forceinline__ float lo_bf16(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float hi_bf16(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ float bf16_at(const __nv_bfloat16* p) {
  return bf16_bits_to_float(__bfloat16_as_ushort(*p));
}

__device__ __forceinline__ void put_bf16(__nv_bfloat16* p, uint32_t bits) {
  *p = __ushort_as_bfloat16(static_cast<unsigned short>(bits));
}

// 32 consecutive bf16 of one row (four 16-byte loads), zero past `valid` columns or when
// `live` is false.  `row` is 16-byte aligned; `valid` columns exist in its padded extent.
__device__ __forceinline__ void load_row32(const __nv_bfloat16* row, int valid, bool live, uint4 (&w)[4]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    if (live && 8 * q < valid)
      w[q] = __ldg(reinterpret_cast<const uint4*>(row) + q);
    else
      w[q] = make_uint4(0u, 0u, 0u, 0u);
  }
  if (live && valid < 32 && valid > 0) {  // ragged tail inside the last loaded chunk
    uint32_t* e = reinterpret_cast<uint32_t*>(w);
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      if (2 * j >= valid) e[j] = 0u;
      else if (2 * j + 1 >= valid) e[j] &= 0xFFFFu;
    }
  }
}

// 32 consecutive bytes of a row of the 8-bit lo buffer (two 16-byte loads); past `valid`
// columns, or when `live` is false, the byte of a zero residual (0x40).  `row` is 16-byte
// aligned.
__device__ __forceinline__ void load_row32_u8(const uint8_t* row, int valid, bool live, uint4 (&w)[2]) {
  constexpr uint32_t kZero4 = 0x40404040u;
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    if (live && 16 * q < valid)
      w[q] = __ldg(reinterpret_cast<const uint4*>(row) + q);
    else
      w[q] = make_uint4(kZero4, kZero4, kZero4, kZero4);
  }
  if (live && valid < 32 && valid > 0) {
    uint32_t* e = reinterpret_cast<uint32_t*>(w);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int k = valid - 4 * j;  // bytes of word j that lie inside the row
      if (k <= 0) e[j] = kZero4;
      else if (k < 4) e[j] = (e[j] & ((1u << (8 * k)) - 1u)) | (kZero4 & ~((1u << (8 * k)) - 1u));
    }
  }
}

// NC (16 or 32) consecutive bf16 of one row (NC / 2 words, element 2i in the low half of
// word i) to `row`, the first `valid` of them only; v8: the segment is 32-byte aligned.
template <int NC>
__device__ __forceinline__ void store_hi_n(__nv_bfloat16* row, int valid, bool v8, const uint32_t (&w)[NC / 2]) {
  if (valid >= NC) {
    if (v8) {
#pragma unroll
      for (int q = 0; q < NC / 16; ++q)
        st_global_v8(row + 16 * q, make_uint4(w[8 * q], w[8 * q + 1], w[8 * q + 2], w[8 * q + 3]),
                     make_uint4(w[8 * q + 4], w[8 * q + 5], w[8 * q + 6], w[8 * q + 7]));
    } else {
#pragma unroll
      for (int q = 0; q < NC / 8; ++q)
        reinterpret_cast<uint4*>(row)[q] = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
    }
  } else {
#pragma unroll
    for (int j = 0; j < NC; ++j)
      if (j < valid) put_bf16(row + j, (j & 1) ? (w[j >> 1] >> 16) : (w[j >> 1] & 0xFFFFu));
  }
}

// NC (16 or 32) stored residual bytes (NC / 4 words, element j in byte j % 4 of word j / 4),
// the first `valid`; v8 (NC = 32): the segment is 32-byte aligned, else 16-byte aligned.
template <int NC>
__device__ __forceinline__ void store_lo_n(uint8_t* row, int valid, bool v8, const uint32_t (&w)[NC / 4]) {
  if (valid >= NC) {
    if (NC == 32 && v8) {
      st_global_v8(row, make_uint4(w[0], w[1], w[2], w[3]), make_uint4(w[4 % (NC / 4)], w[5 % (NC / 4)],
                                                                       w[6 % (NC / 4)], w[7 % (NC / 4)]));
    } else {
#pragma unroll
      for (int q = 0; q < NC / 16; ++q)
        reinterpret_cast<uint4*>(row)[q] = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
    }
  } else {
#pragma unroll
    for (int j = 0; j < NC; ++j)
      if (j < valid) row[j] = static_cast<uint8_t>(w[j >> 2] >> (8 * (j & 3)));
  }
}

// A staged 128-row x 64-byte block of the 8-bit lo buffer (one TMA box, 64-byte swizzle):
// row r at r * 64 B, its 16-byte chunk c (0..3) at chunk c ^ ((r >> 1) & 3).
__device__ __forceinline__ uint32_t lo8_chunk(int r, int c) {
  return static_cast<uint32_t>(r * 64 + ((c ^ ((r >> 1) & 3)) << 4));
}

// Decodes NC values of a row from their bf16 hi and 8-bit lo: the bf16 pairs in `h`
// (NC / 2 words, element 2i in the low half of word i) and the stored residual bytes in
// `l` (NC / 4 words, element j in byte j % 4 of word j / 4).
template <int NC>
__device__ __forceinline__ void decode_row(const uint32_t* h, const uint32_t* l, float (&x)[NC]) {
#pragma unroll
  for (int i = 0; i < NC / 2; ++i) {
    const uint32_t j = 2u * static_cast<uint32_t>(i & 1);
    x[2 * i] = lo8_decode(h[i] << 16, l[i >> 1], j);
    x[2 * i + 1] = lo8_decode(h[i] & 0xFFFF0000u, l[i >> 1], j + 1u);
  }
}

// Stores 128 x 64 staged at Q (two boxes) at rows row0.., columns col0..
__device__ __forceinline__ void store_q(const CUtensorMap* map, const uint8_t* q, int row0, int col0, int mat) {
  tma_store_3d(map, q, col0, row0, mat);
  tma_store_3d(map, q + 8192, col0, row0 + 64, mat);
}

// Stores 64 x 128 staged at T (two boxes side by side) at rows row0.., columns col0..
__device__ __forceinline__ void store_t(const CUtensorMap* map, const uint8_t* t, int row0, int col0, int mat) {
  tma_store_3d(map, t, col0, row0, mat);
  tma_store_3d(map, t + 8192, col0 + 64, row0, mat);
}

// ------------------------------------------------------------------ epilogues

// One 64-column quarter of a symmetric product.  The thread owns row r of this CTA's
// 128-row block and the quarter's columns [32 h, 32 h + 32), whose accumulators start at
// TMEM column tcol.  Off-diagonal block: the row goes to Q and its transpose to T.
// Diagonal block: the whole block goes to Q; the MMA forms (r, c) and (c, r) from the
// same products in the same order, so it is symmetric as computed.
template <int MODE>
__device__ __forceinline__ void sym_quarter(const GemmParams& p, float mul, bool diag, int r, int h, uint32_t tcol,
                                            uint8_t* Q, uint8_t* T, const uint4 (&ain)[4]) {
  uint32_t v[32];
  tmem_ld_32x32b_x32(tcol, v);
  tmem_wait_ld();
  const uint32_t* a = reinterpret_cast<const uint32_t*>(ain);
  uint32_t pk[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    float x0 = __uint_as_float(v[2 * i]), x1 = __uint_as_float(v[2 * i + 1]);
    if (MODE == kPoly) {
      x0 = fmaf(p.c, x0, p.b * lo_bf16(a[i]));
      x1 = fmaf(p.c, x1, p.b * hi_bf16(a[i]));
    } else {
      x0 *= mul;
      x1 *= mul;
    }
    pk[i] = pack_bf16x2(x0, x1);
  }
#pragma unroll
  for (int k = 0; k < 4; ++k)
    *reinterpret_cast<uint4*>(Q + q_chunk(r, 4 * h + k)) = make_uint4(pk[4 * k], pk[4 * k + 1], pk[4 * k + 2], pk[4 * k + 3]);
  if (!diag) {
    // T[c][r], c = 32 h + j: box r / 64, row c, 16-byte chunk ((r & 63) / 8) ^ (c & 7)
    uint8_t* tb = T + ((r >> 6) << 13) + ((r & 7) << 1) + (32 * h) * 128;
    const int rch = (r & 63) >> 3;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const uint32_t bits = (j & 1) ? (pk[j >> 1] >> 16) : (pk[j >> 1] & 0xFFFFu);
      *reinterpret_cast<unsigned short*>(tb + j * 128 + ((rch ^ (j & 7)) << 4)) = static_cast<unsigned short>(bits);
    }
  }
}

// Final epilogue for NC (16 or 32) columns of one row: x holds the orthogonalised update
// for tile columns [c0, c0 + NC) of this CTA's tile row r;  O <- x  and/or
// W <- W decay - lr_scale x.  w_pre: the bf16 W segment, loaded ahead, or nullptr.
template <int MODE, int NC = 32>
__device__ __forceinline__ void write_update(const FinalParams& p, const ClassDesc& cd, const Tile& tl, int rank,
                                             int r, int c0, const float (&x)[NC], const uint4* w_pre = nullptr) {
  const int R = Lay<MODE>::TM * tl.I + kBM * rank + r;
  const int C0 = Lay<MODE>::TN * tl.J + c0;
  const int cols = cd.cols;
  if (R >= cd.rows || C0 >= cols) return;
  const bool full = C0 + NC <= cols;
  const UpdMat& u = p.upd[cd.mat_base + tl.mat];
  if (u.out != nullptr) {
    float* o = u.out + static_cast<int64_t>(R) * cols + C0;
    if (full && u.vec_out == 2) {
#pragma unroll
      for (int q = 0; q < NC / 8; ++q)
        st_global_v8(o + 8 * q,
                     make_uint4(__float_as_uint(x[8 * q]), __float_as_uint(x[8 * q + 1]), __float_as_uint(x[8 * q + 2]),
                                __float_as_uint(x[8 * q + 3])),
                     make_uint4(__float_as_uint(x[8 * q + 4]), __float_as_uint(x[8 * q + 5]),
                                __float_as_uint(x[8 * q + 6]), __float_as_uint(x[8 * q + 7])));
    } else if (full && u.vec_out) {
#pragma unroll
      for (int q = 0; q < NC / 4; ++q)
        reinterpret_cast<float4*>(o)[q] = make_float4(x[4 * q], x[4 * q + 1], x[4 * q + 2], x[4 * q + 3]);
    } else {
#pragma unroll
      for (int j = 0; j < NC; ++j)
        if (C0 + j < cols) o[j] = x[j];
    }
  }
  if (u.param != nullptr) {
    const float decay = p.decay, ls = u.lr_scale;
    if (u.param_bf16) {
      __nv_bfloat16* w = static_cast<__nv_bfloat16*>(u.param) + static_cast<int64_t>(R) * u.ld_param + C0;
      if (full && u.vec_param) {
        const bool v8 = u.vec_param == 2;  // 32-byte rows: 256-bit accesses
        uint4 raw[NC / 8];
        if (w_pre != nullptr) {
#pragma unroll
          for (int q = 0; q < NC / 8; ++q) raw[q] = w_pre[q];
        } else if (v8) {
#pragma unroll
          for (int q = 0; q < NC / 16; ++q) ld_global_v8(w + 16 * q, raw[2 * q], raw[2 * q + 1]);
        } else {
#pragma unroll
          for (int q = 0; q < NC / 8; ++q) raw[q] = reinterpret_cast<const uint4*>(w)[q];
        }
        const uint32_t* rw = reinterpret_cast<const uint32_t*>(raw);
        uint32_t wb[NC / 2];
#pragma unroll
        for (int i = 0; i < NC / 2; ++i)
          wb[i] = pack_bf16x2(fmaf(-ls, x[2 * i], lo_bf16(rw[i]) * decay), fmaf(-ls, x[2 * i + 1], hi_bf16(rw[i]) * decay));
        if (v8) {
#pragma unroll
          for (int q = 0; q < NC / 16; ++q)
            st_global_v8(w + 16 * q, make_uint4(wb[8 * q], wb[8 * q + 1], wb[8 * q + 2], wb[8 * q + 3]),
                         make_uint4(wb[8 * q + 4], wb[8 * q + 5], wb[8 * q + 6], wb[8 * q + 7]));
        } else {
#pragma unroll
          for (int q = 0; q < NC / 8; ++q)
            reinterpret_cast<uint4*>(w)[q] = make_uint4(wb[4 * q], wb[4 * q + 1], wb[4 * q + 2], wb[4 * q + 3]);
        }
      } else {
#pragma unroll
        for (int j = 0; j < NC; ++j)
          if (C0 + j < cols) put_bf16(w + j, float_to_bf16_bits(fmaf(-ls, x[j], bf16_at(w + j) * decay)));
      }
    } else {
      float* w = static_cast<float*>(u.param) + static_cast<int64_t>(R) * u.ld_param + C0;
      if (full && u.vec_param == 2) {
#pragma unroll
        for (int q = 0; q < NC / 8; ++q) {
          uint4 a, b;
          ld_global_v8(w + 8 * q, a, b);
          const uint32_t in[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
          uint32_t out[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) out[j] = __float_as_uint(fmaf(-ls, x[8 * q + j], __uint_as_float(in[j]) * decay));
          st_global_v8(w + 8 * q, make_uint4(out[0], out[1], out[2], out[3]), make_uint4(out[4], out[5], out[6], out[7]));
        }
      } else if (full && u.vec_param) {
#pragma unroll
        for (int q = 0; q < NC / 4; ++q) {
          float4 t = reinterpret_cast<float4*>(w)[q];
          t.x = fmaf(-ls, x[4 * q], t.x * decay);
          t.y = fmaf(-ls, x[4 * q + 1], t.y * decay);
          t.z = fmaf(-ls, x[4 * q + 2], t.z * decay);
          t.w = fmaf(-ls, x[4 * q + 3], t.w * decay);
          reinterpret_cast<float4*>(w)[q] = t;
        }
      } else {
#pragma unroll
        for (int j = 0; j < NC; ++j)
          if (C0 + j < cols) w[j] = fmaf(-ls, x[j], w[j] * decay);
      }
    }
  }
}

// The bf16 W row segment write_update<MODE, NC> reads for tile columns [c0, c0 + NC) of
// this CTA's tile row r, loaded ahead of time; false where write_update takes another path.
template <int MODE, int NC>
__device__ __forceinline__ bool load_w_segment(const FinalParams& p, const ClassDesc& cd, const Tile& tl, int rank,
                                               int r, int c0, uint4 (&w)[NC / 8]) {
  const UpdMat& u = p.upd[cd.mat_base + tl.mat];
  const int R = Lay<MODE>::TM * tl.I + kBM * rank + r;
  const int C0 = Lay<MODE>::TN * tl.J + c0;
  if (u.param == nullptr || !u.param_bf16 || !u.vec_param || R >= cd.rows || C0 + NC > cd.cols) return false;
  const __nv_bfloat16* row = static_cast<const __nv_bfloat16*>(u.param) + static_cast<int64_t>(R) * u.ld_param + C0;
  if (u.vec_param == 2) {  // 32-byte rows: 256-bit loads
#pragma unroll
    for (int q = 0; q < NC / 16; ++q) ld_global_v8(row + 16 * q, w[2 * q], w[2 * q + 1]);
  } else {
#pragma unroll
    for (int q = 0; q < NC / 8; ++q) w[q] = reinterpret_cast<const uint4*>(row)[q];
  }
  return true;
}

// X update for the 32 tile columns [c0, c0 + 32) of this CTA's tile row r, with the old
// hi (16 bf16x2 words) and lo (8 words of residual bytes) already in registers:
// x = s (a (hi + lo) + acc).  kApply returns the new pair packed (hb: 16 bf16x2 words,
// lb: 8 words of bytes); kApplyLast updates W and/or writes O in global memory.
template <int MODE>
__device__ __forceinline__ void apply_quarter(const typename ParamsOf<MODE>::type& p, const ClassDesc& cd,
                                              const Tile& tl, int rank, int r, int c0, uint32_t tcol,
                                              const uint4 (&xh4)[4], const uint4 (&xl4)[2], float s,
                                              uint32_t (&hb)[16], uint32_t (&lb)[8], const uint4* w_pre = nullptr) {
  uint32_t v[32];
  tmem_ld_32x32b_x32(tcol, v);
  float x[32];
  decode_row<32>(reinterpret_cast<const uint32_t*>(xh4), reinterpret_cast<const uint32_t*>(xl4), x);
  tmem_wait_ld();
#pragma unroll
  for (int j = 0; j < 32; ++j) x[j] = s * fmaf(p.a, x[j], __uint_as_float(v[j]));
  if constexpr (MODE == kApply) {
#pragma unroll
    for (int k = 0; k < 8; ++k)
      split_hi_lo8x4(x[4 * k], x[4 * k + 1], x[4 * k + 2], x[4 * k + 3], hb[2 * k], hb[2 * k + 1], lb[k]);
  } else {
    (void)hb;
    (void)lb;
    write_update<MODE>(p, cd, tl, rank, r, c0, x, w_pre);
  }
}

template <int NC>
__device__ __forceinline__ void tmem_ld_row(uint32_t taddr, uint32_t (&v)[NC]) {
  if constexpr (NC == 32)
    tmem_ld_32x32b_x32(taddr, v);
  else
    tmem_ld_32x32b_x16(taddr, v);
}

// ------------------------------------------------------------------ the kernel

template <int MODE, int VAR>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(Lay<MODE, VAR>::kThreads, 1)
    muon_ns_gemm_kernel(const __grid_constant__ typename ParamsOf<MODE>::type p) {
  using L = Lay<MODE, VAR>;
  constexpr bool SMALL = L::SMALL;
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
  uint64_t* efull = tdown + 1;  // staged variant: quarter q of the tile's hi/lo inputs has landed
  uint64_t* pdone = efull + 4;  // used in the leader CTA: the peer's producer has finished
  uint64_t* consumed = pdone + 1;  // staged apply: every epilogue warp has read quarter q
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(consumed + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* epi_flag = abort_flag + 1;
  volatile uint32_t* peer_issued = reinterpret_cast<volatile uint32_t*>(epi_flag + 1);  // leader CTA

  griddep_launch_dependents();
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
    for (int q = 0; q < 4; ++q) mbar_init(&efull[q], 1);
    mbar_init(pdone, 1);
    for (int q = 0; q < 4; ++q) mbar_init(&consumed[q], L::NEPI);
    *abort_flag = 0;
    *epi_flag = 1;  // live; an epilogue wait that gives up clears it
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    for (int c = 0; c < p.num_classes; ++c) {
      tma_prefetch_desc(&p.map_a[c]);
      tma_prefetch_desc(&p.map_b[c]);
      if (VAR != kStreamed) {
        tma_prefetch_desc(&p.map_in[c]);
        tma_prefetch_desc(&p.map_out2[c]);
      }
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
  griddep_wait();  // operands and scales come from the previous kernel of the step

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer (both CTAs)
    // Stage-loads are numbered in issue order; load i uses stage i % S in phase i / S.  The
    // leader arms each phase for both CTAs' bytes.  After a timeout the two producers may
    // stop at different counts, so the peer reports its count and the leader settles every
    // phase still open before the CTAs part (see settle below).
    if (lane == 0) {
      const uint32_t full0 = map_to_rank(smem_u32(full), 0);
      int s = 0;
      uint32_t ph = 0;
      uint32_t issued = 0;
      bool ok = true;
      for (int t = pair; ok && t < p.total_tiles; t += npairs) {
        const Tile tl = decode_tile<MODE>(p, t);
        const ClassDesc& cd = p.cls[tl.cls];
        const CUtensorMap* ma = &p.map_a[tl.cls];
        const CUtensorMap* mb = &p.map_b[tl.cls];
        const int nk = (cd.ksize + L::BK - 1) / L::BK;
        const int a0 = L::TM * tl.I + kBM * rank;
        const int b0 = L::TN * tl.J + kBM * rank;
        const bool diag = is_diag_tile<MODE>(tl);
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&empty[s], ph ^ 1u, wd, kSiteProducerEmpty)) {
            ok = false;
            break;
          }
          uint8_t* sa = smem + s * L::kStageBytes;
          uint8_t* sb = sa + L::kABytes;
          if (leader_cta) mbar_arrive_expect_tx(&full[s], 2 * (diag ? L::kABytes : L::kStageBytes));
          const uint32_t fb = full0 + 8u * static_cast<uint32_t>(s);
          const int k0 = kb * L::BK;
          load_operand_pair<L::BK>(sa, ma, cd.a_mn, a0, k0, tl.mat, fb);
          if (!diag) load_operand_pair<L::BK>(sb, mb, cd.b_mn, b0, k0, tl.mat, fb);
          ++issued;
          if (++s == S) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
      if (!leader_cta) {
        st_cluster_u32(map_to_rank(smem_u32(const_cast<uint32_t*>(peer_issued)), 0), issued);
        mbar_arrive_cluster(map_to_rank(smem_u32(pdone), 0));
      } else {
        // Settle.  A load i below min(nL, nP) - S has completed: both producers waited for
        // stage i % S to be consumed again.  Each remaining i, in order, is waited for after
        //   i < nL, i < nP : nothing (armed, both shares issued)
        //   i < nL, i >= nP: completing the peer's share, which will never be sent
        //   i >= nL, i < nP: arming the phase for the peer's share alone
        // so no copy is in flight into either CTA when the final cluster barrier opens.
        // Phase i of a stage completes before load i + S of it is issued, so every wait
        // below is for the stage's current phase.
        const uint32_t nl = issued;
        uint32_t np = nl;
        bool known = false;
        {
          const uint64_t t0 = global_timer_ns();
          while (!(known = mbar_try_wait_cluster(pdone, 0)) && global_timer_ns() - t0 < tb) {
          }
          if (known) np = *peer_issued;
        }
        const uint32_t both = nl < np ? nl : np;
        const uint32_t lo_i = both >= static_cast<uint32_t>(S) ? both - S : 0u;
        const uint32_t hi_i = nl > np ? nl : np;
        for (uint32_t i = lo_i; i < hi_i; ++i) {
          const int st = static_cast<int>(i % S);
          const uint32_t par = (i / S) & 1u;
          if (i >= nl)
            mbar_arrive_expect_tx(&full[st], load_share_bytes<MODE, L>(p, pair, npairs, i));
          else if (i >= np)
            mbar_complete_tx(&full[st], load_share_bytes<MODE, L>(p, pair, npairs, i));
          quiet_wait(&full[st], par, tb);
        }
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
          const int nk = (cd.ksize + L::BK - 1) / L::BK;
          const uint32_t idesc = idesc_bf16_f32(L::TM, L::TN, cd.a_mn, cd.b_mn);
          const bool diag = is_diag_tile<MODE>(tl);
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
            const uint32_t sb = diag ? sa : sa + L::kABytes;
#pragma unroll
            for (int kk = 0; kk < L::BK / 16; ++kk)
              umma_bf16_pair(dtm, operand_desc<L::BK>(sa, cd.a_mn, kk), operand_desc<L::BK>(sb, cd.b_mn, kk), idesc,
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
  } else if (L::kLoader && warp == L::kLoaderWarp) {
    // ---------------------------------------------------------------- epilogue input loader (both CTAs)
    // The quarters of this pair's tiles, in order (quarter g = 4 k + q of the k-th tile), go
    // to slot g % kSlots: this CTA's 128 rows x 64 columns of the old hi and lo, loaded once
    // every epilogue warp has read quarter g - kSlots from that slot.  (Prefetching the next
    // tile's quarters into L2 at the start of each tile measured slower.)
    if (lane == 0) {
      constexpr int NS = L::kSlots > 0 ? L::kSlots : 1;  // (this branch runs in the staged applies only)
      int k = 0;
      uint32_t g = 0;
      bool ok = true;
      uint32_t issued = 0, last_par = 0;  // per slot: a load issued; the parity of the last one
      for (int t = pair; ok && t < p.total_tiles; t += npairs, ++k) {
        const Tile tl = decode_tile<MODE>(p, t);
        const int row0 = L::TM * tl.I + kBM * rank, col0 = L::TN * tl.J;
        for (int q = 0; q < 4; ++q, ++g) {
          const int sl = static_cast<int>(g % NS);
          if (g >= static_cast<uint32_t>(NS) &&
              !mbar_wait(&consumed[sl], ((g / NS) - 1u) & 1u, wd, kSiteProducerEpi)) {
            ok = false;
            break;
          }
          uint8_t* slot = epi + sl * L::kSlotBytes;
          mbar_arrive_expect_tx(&efull[sl], L::kSlotBytes);
          tma_load_3d(slot, &p.map_in[tl.cls], &efull[sl], col0 + 64 * q, row0, tl.mat);
          tma_load_3d(slot + L::kBox64, &p.map_in[tl.cls], &efull[sl], col0 + 64 * q, row0 + 64, tl.mat);
          tma_load_3d(slot + 2 * L::kBox64, &p.map_out2[tl.cls], &efull[sl], col0 + 64 * q, row0, tl.mat);
          issued |= 1u << sl;
          last_par = (last_par & ~(1u << sl)) | (((g / NS) & 1u) << sl);
        }
      }
      // Before the CTA leaves, every load issued has landed.  A slot has at most one load
      // outstanding: the one before it was waited for by every epilogue warp.
      for (int sl = 0; sl < NS; ++sl)
        if (issued & (1u << sl)) quiet_wait(&efull[sl], (last_par >> sl) & 1u, tb);
    }
  } else if constexpr (SMALL && !kSym) {
    // ---------------------------------------------------------------- staged apply epilogue (both CTAs)
    // The tile's old hi and lo (128 x 256 each per CTA) arrive in shared memory as 64-column
    // quarters from the loader warp, quarter g of this pair's sequence in slot g % kSlots.
    // Each warp waits for the accumulator and each quarter itself, reads its part, tells the
    // loader it is done with the slot, and writes its results straight to global memory:
    // the new pair (kApply) or W and/or O (kApplyLast).  The epilogue warps never wait for
    // one another.
    const int ew = warp - 2;
    const int q4 = warp & 3;  // TMEM lanes 32 q4 .. 32 q4 + 31 belong to this warp
    constexpr int NC = 256 / L::NEPI;  // columns of each quarter per thread
    const int h = ew >> 2;             // which NC columns of each 64-column quarter
    const int r = q4 * 32 + lane;
    const uint32_t tempty0 = map_to_rank(smem_u32(tempty), 0);
    constexpr int NS = L::kSlots;
    int acc = 0;
    uint32_t aph = 0;
    uint32_t g = 0;  // quarters of this pair's tiles so far
    for (int t = pair; t < p.total_tiles; t += npairs) {
      const Tile tl = decode_tile<MODE>(p, t);
      const ClassDesc& cd = p.cls[tl.cls];
      const int Rx = L::TM * tl.I + kBM * rank + r;
      const bool live = Rx < cd.rows;
      const bool hv8 = (cd.ldx & 15) == 0, lv8 = (cd.ldl & 31) == 0;  // 32-byte rows
      const int64_t xoff = tl.mat * cd.x_stride + static_cast<int64_t>(Rx) * cd.ldx;
      const int64_t loff = tl.mat * cd.lo_stride + static_cast<int64_t>(Rx) * cd.ldl;
      const float sc = p.first_iter ? p.scale[cd.mat_base + tl.mat] : 1.f;
      const uint32_t tacc = tmem_base + static_cast<uint32_t>(acc * L::TN) + (static_cast<uint32_t>(q4 * 32) << 16);
      uint4 wq[NC / 8];
      bool wq_ok = false;
      if constexpr (MODE == kApplyLast) {
        wq_ok = load_w_segment<MODE, NC>(p, cd, tl, rank, r, NC * h, wq);
        if (h == 0 && t + npairs < p.total_tiles) {  // warm L2 with this thread's row of W in the next tile
          const Tile nx = decode_tile<MODE>(p, t + npairs);
          const ClassDesc& nd = p.cls[nx.cls];
          const UpdMat& un = p.upd[nd.mat_base + nx.mat];
          const int Rn = L::TM * nx.I + kBM * rank + r, Cn = L::TN * nx.J;
          if (un.param != nullptr && Rn < nd.rows) {
            const int esz = un.param_bf16 ? 2 : 4;
            const int bytes = (nd.cols - Cn < L::TN ? nd.cols - Cn : L::TN) * esz;
            const char* row = static_cast<const char*>(un.param) + (static_cast<int64_t>(Rn) * un.ld_param + Cn) * esz;
            for (int off = 0; off < bytes; off += 128) prefetch_l2(row + off);
            prefetch_l2(row + bytes - 1);
          }
        }
      }
      bool ok = warp_wait(&tfull[acc], aph, wd, kSiteEpilogueFull);
      if (ok) tc_fence_after();
#pragma unroll 1
      for (int q = 0; ok && q < 4; ++q, ++g) {
        const int sl = static_cast<int>(g % NS);
        ok = warp_wait(&efull[sl], (g / NS) & 1u, wd, kSiteEpilogueIn);
        if (!ok) break;
        const uint8_t* slot = epi + sl * L::kSlotBytes;
        const int c0 = 64 * q + NC * h;
        uint4 wn[NC / 8];
        bool wn_ok = false;
        if constexpr (MODE == kApplyLast) wn_ok = q < 3 && load_w_segment<MODE, NC>(p, cd, tl, rank, r, c0 + 64, wn);
        uint32_t v[NC];
        tmem_ld_row<NC>(tacc + c0, v);
        uint4 xh4[NC / 8], xl4[NC / 16];
#pragma unroll
        for (int i = 0; i < NC / 8; ++i)
          xh4[i] = *reinterpret_cast<const uint4*>(slot + quarter_chunk(r, (NC / 8) * h + i));
        const uint8_t* lq = slot + 2 * L::kBox64;
#pragma unroll
        for (int i = 0; i < NC / 16; ++i) xl4[i] = *reinterpret_cast<const uint4*>(lq + lo8_chunk(r, (NC / 16) * h + i));
        float x[NC];
        decode_row<NC>(reinterpret_cast<const uint32_t*>(xh4), reinterpret_cast<const uint32_t*>(xl4), x);
        tmem_wait_ld();  // before any other asm: v is written asynchronously until here
        // The slot may be refilled once every warp's reads of it have completed: the decode
        // above consumed the loaded values, and the proxy fence orders these generic-proxy
        // reads before the loader's TMA (async-proxy) write of the next tile's quarter.
        // (Without the fence the loader's refill was measured to race these reads.)
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&consumed[sl]);  // this warp is done with the slot
        if (q == 3) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster_relaxed(tempty0 + 8u * static_cast<uint32_t>(acc));
        }
#pragma unroll
        for (int j = 0; j < NC; ++j) x[j] = fmaf(p.a, x[j], __uint_as_float(v[j]));
        if (sc != 1.f) {  // iteration 0 only (uniform)
#pragma unroll
          for (int j = 0; j < NC; ++j) x[j] *= sc;
        }
        if constexpr (MODE == kApply) {
          uint32_t hb[NC / 2], lb[NC / 4];
#pragma unroll
          for (int i = 0; i < NC / 4; ++i)
            split_hi_lo8x4(x[4 * i], x[4 * i + 1], x[4 * i + 2], x[4 * i + 3], hb[2 * i], hb[2 * i + 1], lb[i]);
          const int C = L::TN * tl.J + c0;
          store_hi_n<NC>(cd.x_hi_next + xoff + C, live ? cd.cols - C : 0, hv8, hb);
          store_lo_n<NC>(cd.x_lo + loff + C, live ? cd.cols - C : 0, lv8, lb);
        } else {
          write_update<MODE, NC>(p, cd, tl, rank, r, c0, x, wq_ok ? wq : nullptr);
#pragma unroll
          for (int i = 0; i < NC / 8; ++i) wq[i] = wn[i];
          wq_ok = wn_ok;
        }
      }
      if (!ok) break;
      if (++acc == 2) {
        acc = 0;
        aph ^= 1u;
      }
    }
  } else if constexpr (SMALL) {
    // ---------------------------------------------------------------- staged symmetric epilogue (both CTAs)
    // Output quarters alternate between two staging buffers, so the TMA stores of one
    // drain while the next is written.  The polynomial's A block is staged like the
    // apply's inputs: four 64-column quarters, each refilled for the next tile as soon as
    // it has been read.
    const int ew = warp - 2;
    const int q4 = warp & 3;
    const int h = ew >> 2;
    const int r = q4 * 32 + lane;
    const bool leader = threadIdx.x == 64;  // also the thread that waits on the barriers
    const uint32_t tempty0 = map_to_rank(smem_u32(tempty), 0);
    uint8_t* Ain = epi + 2 * L::kOutBufs * L::kHalf;
    int acc = 0;
    uint32_t aph = 0;
    uint32_t pending = 0, pend_par = 0;
    uint32_t used = 0;  // output quarters handed to TMA stores so far (uniform)
    auto load_quarter = [&](const Tile& nx, int q, uint32_t par) {
      mbar_arrive_expect_tx(&efull[q], L::kHalf);
      load_region_quarter(Ain, &p.map_in[nx.cls], &efull[q], q, L::TM * nx.I + kBM * rank, L::TN * nx.J, nx.mat);
      pending |= 1u << q;
      pend_par = (pend_par & ~(1u << q)) | (par << q);
    };
    constexpr bool kStageA = MODE == kPoly;
    if (kStageA && leader && pair < p.total_tiles) {
      const Tile first = decode_tile<MODE>(p, pair);
      for (int q = 0; q < 4; ++q) load_quarter(first, q, 0u);
    }
    int k = 0;
    bool live = true;
    for (int t = pair; live && t < p.total_tiles; t += npairs, ++k) {
      const Tile tl = decode_tile<MODE>(p, t);
      const ClassDesc& cd = p.cls[tl.cls];
      const uint32_t kpar = static_cast<uint32_t>(k) & 1u;
      const bool has_next = t + npairs < p.total_tiles;
      Tile nx = tl;
      if (has_next) nx = decode_tile<MODE>(p, t + npairs);
      const int rb = 2 * tl.I + rank;
      float mul = 1.f;
      if (MODE == kGram && p.first_iter) {
        const float sv = p.scale[cd.mat_base + tl.mat];
        mul = sv * sv;
      }
      const uint32_t tacc = tmem_base + static_cast<uint32_t>(acc * L::TN) + (static_cast<uint32_t>(q4 * 32) << 16);
#pragma unroll 1
      for (int q = 0; q < 4; ++q) {
        const int cb = 2 * tl.J + (q >> 1);
        const bool skip = rb > cb;  // below the diagonal: stored by the block's mirror (uniform)
        if (ew == 0) {
          bool ok = q > 0 || warp_wait(&tfull[acc], aph, wd, kSiteEpilogueFull);
          if (kStageA && ok) ok = warp_wait(&efull[q], kpar, wd, kSiteEpilogueIn);
          if (lane == 0) {
            *epi_flag = ok ? 1 : 0;
            if (ok) pending &= ~(1u << q);
            if (!skip) {  // the stores that used this buffer last have read it
              if constexpr (L::kOutBufs == 1) bulk_wait_read<0>();
              else bulk_wait_read<1>();
            }
          }
        }
        named_barrier(1, NT);
        if (*epi_flag == 0) {
          live = false;
          break;
        }
        if (q == 0) tc_fence_after();
        if (!skip) {
          uint8_t* Q = epi + (L::kOutBufs == 1 ? 0u : (used & 1u)) * (2 * L::kHalf);
          uint8_t* Tst = Q + L::kHalf;
          uint4 ain[4];
#pragma unroll
          for (int i = 0; i < 4; ++i)
            ain[i] = MODE == kPoly ? *reinterpret_cast<const uint4*>(Ain + region_chunk(r, 8 * q + 4 * h + i))
                                   : make_uint4(0u, 0u, 0u, 0u);
          sym_quarter<MODE>(p, mul, rb == cb, r, h, tacc + 64 * q + 32 * h, Q, Tst, ain);
          fence_proxy_async_smem();
          named_barrier(1, NT);
          if (leader) {
            store_q(&p.map_out[tl.cls], Q, kBM * rb, kBM * cb + 64 * (q & 1), tl.mat);
            if (rb != cb) store_t(&p.map_out[tl.cls], Tst, kBM * cb + 64 * (q & 1), kBM * rb, tl.mat);
            bulk_commit();
          }
          ++used;
        }
        if (q == 3) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster_relaxed(tempty0 + 8u * static_cast<uint32_t>(acc));
        }
        if (kStageA && leader && has_next) load_quarter(nx, q, kpar ^ 1u);
      }
      if (!live) break;
      if (++acc == 2) {
        acc = 0;
        aph ^= 1u;
      }
    }
    if (leader) {
      bulk_wait_all();
      for (int q = 0; q < 4; ++q)
        if (pending & (1u << q)) quiet_wait(&efull[q], (pend_par >> q) & 1u, tb);
    }
  } else {
    // ---------------------------------------------------------------- epilogue (both CTAs)
    const int ew = warp - 2;
    const int q4 = warp & 3;  // TMEM lanes 32 q4 .. 32 q4 + 31 belong to this warp
    const int h = ew >> 2;    // which 32 columns of each 64-column quarter
    const int r = q4 * 32 + lane;
    const bool leader = threadIdx.x == 64;
    const uint32_t tempty0 = map_to_rank(smem_u32(tempty), 0);
    uint8_t* Q = epi;
    uint8_t* Tst = epi + L::kHalf;
    int acc = 0;
    uint32_t aph = 0;
    for (int t = pair; t < p.total_tiles; t += npairs) {
      const Tile tl = decode_tile<MODE>(p, t);
      const ClassDesc& cd = p.cls[tl.cls];
      // Epilogue inputs come straight from global memory (L2) into registers; they are
      // requested before the accumulator is waited for.
      uint4 in_a[4][4];  // polynomial: A, the four quarters' 32 columns of this row
      uint4 ch[4], cl[2];  // apply: hi and 8-bit lo of the first quarter
      const int rb = 2 * tl.I + rank;
      const int Rx = L::TM * tl.I + kBM * rank + r;
      const int64_t xoff = tl.mat * cd.x_stride + static_cast<int64_t>(Rx) * cd.ldx;
      const int64_t loff = tl.mat * cd.lo_stride + static_cast<int64_t>(Rx) * cd.ldl;
      const int Cb = L::TN * tl.J + 32 * h;
      if constexpr (MODE == kPoly) {
        const int Ra = kBM * rb + r;
        const __nv_bfloat16* arow = cd.a_buf + tl.mat * cd.a_stride + static_cast<int64_t>(Ra) * cd.lda;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int cb = 2 * tl.J + (q >> 1);
          const int C = Cb + 64 * q;
          load_row32(arow + C, cd.m - C, Ra < cd.m && rb <= cb, in_a[q]);
        }
      } else if constexpr (!kSym) {
        load_row32(cd.x_hi_cur + xoff + Cb, cd.cols - Cb, Rx < cd.rows, ch);
        load_row32_u8(cd.x_lo + loff + Cb, cd.cols - Cb, Rx < cd.rows, cl);
      }
      // The next tile's epilogue inputs start moving from HBM into L2 now, so that its
      // loads above hit L2 (apply: hi and lo; polynomial: A).
      if (MODE != kGram && leader && t + npairs < p.total_tiles) {
        const Tile nx = decode_tile<MODE>(p, t + npairs);
        const ClassDesc& nd = p.cls[nx.cls];
        if constexpr (MODE == kPoly) {
          const int rbn = 2 * nx.I + rank;
#pragma unroll
          for (int c = 0; c < 4; ++c) tma_prefetch_l2_3d(&p.map_a[nx.cls], L::TN * nx.J + 64 * c, kBM * rbn, nx.mat);
        } else {
          const int rn = L::TM * nx.I + kBM * rank;
          const CUtensorMap* mh = nd.tall ? &p.map_a[nx.cls] : &p.map_b[nx.cls];  // the operand map of hi
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            tma_prefetch_l2_3d(mh, L::TN * nx.J + 64 * c, rn, nx.mat);
            tma_prefetch_l2_3d(&p.map_out2[nx.cls], L::TN * nx.J + 64 * c, rn, nx.mat);  // 128 rows of lo
          }
        }
      }
      // One warp waits for the accumulator; the rest learn the outcome at the barrier, so
      // every epilogue warp leaves the loop together.
      if (ew == 0) {
        const bool ok = warp_wait(&tfull[acc], aph, wd, kSiteEpilogueFull);
        if (lane == 0) *epi_flag = ok ? 1 : 0;
      }
      named_barrier(1, NT);
      if (*epi_flag == 0) break;
      tc_fence_after();
      const uint32_t tacc = tmem_base + static_cast<uint32_t>(acc * L::TN) + (static_cast<uint32_t>(q4 * 32) << 16);
      if constexpr (kSym) {
        float mul = 1.f;
        if (MODE == kGram && p.first_iter) {
          const float sv = p.scale[cd.mat_base + tl.mat];
          mul = sv * sv;
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int cb = 2 * tl.J + (q >> 1);
          if (rb > cb) continue;  // below the diagonal: stored by the block's mirror
          if (leader) bulk_wait_read<0>();
          named_barrier(1, NT);  // staging free
          sym_quarter<MODE>(p, mul, rb == cb, r, h, tacc + 64 * q + 32 * h, Q, Tst, in_a[q]);
          if (q == 3) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster_relaxed(tempty0 + 8u * static_cast<uint32_t>(acc));
          }
          fence_proxy_async_smem();
          named_barrier(1, NT);
          if (leader) {
            store_q(&p.map_out[tl.cls], Q, kBM * rb, kBM * cb + 64 * (q & 1), tl.mat);
            if (rb != cb) store_t(&p.map_out[tl.cls], Tst, kBM * cb + 64 * (q & 1), kBM * rb, tl.mat);
            bulk_commit();
          }
        }
      } else {
        const float sc = p.first_iter ? p.scale[cd.mat_base + tl.mat] : 1.f;
        const int row0 = L::TM * tl.I + kBM * rank;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint4 nh[4], nl[2];
          if (q < 3) {
            const int Cn = Cb + 64 * (q + 1);
            load_row32(cd.x_hi_cur + xoff + Cn, cd.cols - Cn, Rx < cd.rows, nh);
            load_row32_u8(cd.x_lo + loff + Cn, cd.cols - Cn, Rx < cd.rows, nl);
          }
          uint32_t hb[16], lb[8];
          apply_quarter<MODE>(p, cd, tl, rank, r, 64 * q + 32 * h, tacc + 64 * q + 32 * h, ch, cl, sc, hb, lb);
          if (q == 3) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster_relaxed(tempty0 + 8u * static_cast<uint32_t>(acc));
          }
          if constexpr (MODE == kApply) {
            if (leader) bulk_wait_read<0>();
            named_barrier(1, NT);  // staging free
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const uint32_t o = q_chunk(r, 4 * h + k);
              *reinterpret_cast<uint4*>(Q + o) = make_uint4(hb[4 * k], hb[4 * k + 1], hb[4 * k + 2], hb[4 * k + 3]);
            }
            // the quarter's 8-bit lo: one 128-row x 64-byte block at Tst, chunks 2 h, 2 h + 1
#pragma unroll
            for (int k = 0; k < 2; ++k)
              *reinterpret_cast<uint4*>(Tst + lo8_chunk(r, 2 * h + k)) =
                  make_uint4(lb[4 * k], lb[4 * k + 1], lb[4 * k + 2], lb[4 * k + 3]);
            fence_proxy_async_smem();
            named_barrier(1, NT);
            if (leader) {
              store_q(&p.map_out[tl.cls], Q, row0, L::TN * tl.J + 64 * q, tl.mat);
              tma_store_3d(&p.map_out2[tl.cls], Tst, L::TN * tl.J + 64 * q, row0, tl.mat);
              bulk_commit();
            }
          }
          if (q < 3) {
#pragma unroll
            for (int k = 0; k < 4; ++k) ch[k] = nh[k];
#pragma unroll
            for (int k = 0; k < 2; ++k) cl[k] = nl[k];
          }
        }
      }
      if (++acc == 2) {
        acc = 0;
        aph ^= 1u;
      }
    }
    if (leader) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // nothing arrives on, or lands in, either CTA after this point
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, L::kTmemCols);
  }
}

template <int MODE, int VAR>
static cudaError_t launch_one(const typename ParamsOf<MODE>::type& p, int max_pairs, cudaStream_t stream) {
  using L = Lay<MODE, VAR>;
  auto* kernel = muon_ns_gemm_kernel<MODE, VAR>;
  static thread_local int configured_device = -1;
  static thread_local int resident_pairs = 0;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (configured_device != dev) {
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kSmemBytes);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * max_pairs, 1, 1);
    cfg.blockDim = dim3(L::kThreads, 1, 1);
    cfg.dynamicSmemBytes = L::kSmemBytes;
    int clusters = 0;
    e = cudaOccupancyMaxActiveClusters(&clusters, kernel, &cfg);
    if (e != cudaSuccess) return e;
    resident_pairs = clusters > 0 ? clusters : 1;
    configured_device = dev;
  }
  const int pairs = std::max(1, std::min(std::min(p.total_tiles, max_pairs), resident_pairs));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs, 1, 1);
  cfg.blockDim = dim3(L::kThreads, 1, 1);
  cfg.dynamicSmemBytes = L::kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, p);
}

int gemm_tile_rows() { return 256; }
int gemm_tile_cols() { return 256; }

// `max_pairs` bounds the number of CTA pairs (half the SM count).  Apply launches with
// p->staged set run the staged variant, whose operand maps have 64 x 64 boxes.
cudaError_t launch_gemm(int mode, const GemmParams* p, int max_pairs, cudaStream_t stream) {
  switch (mode) {
    case kGram:
      return p->staged == kStaged ? launch_one<kGram, kStaged>(*p, max_pairs, stream)
                                  : launch_one<kGram, kStreamed>(*p, max_pairs, stream);
    case kPoly:
      return p->staged == kStaged ? launch_one<kPoly, kStaged>(*p, max_pairs, stream)
                                  : launch_one<kPoly, kStreamed>(*p, max_pairs, stream);
    case kApply:
      return p->staged == kStaged ? launch_one<kApply, kStaged>(*p, max_pairs, stream)
                                  : launch_one<kApply, kStreamed>(*p, max_pairs, stream);
    case kApplyLast: {
      const FinalParams& f = *static_cast<const FinalParams*>(p);
      return p->staged == kStaged ? launch_one<kApplyLast, kStaged>(f, max_pairs, stream)
                                  : launch_one<kApplyLast, kStreamed>(f, max_pairs, stream);
    }
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace muon
