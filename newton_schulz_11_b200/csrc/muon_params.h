// Launch parameter blocks shared by the host planner and the kernels.
//
// Everything a kernel needs travels by value in its parameter block
// (__grid_constant__), so a step can be captured in a CUDA graph and no
// per-call host-to-device copy is needed.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <stdint.h>

namespace muon {

constexpr int kMaxClasses = 8;      // distinct shapes per wave
constexpr int kMaxWaveMats = 128;   // matrices per wave
constexpr int kBM = 128;            // tile rows = UMMA M
constexpr int kBox = 64;            // TMA box inner edge (elements, 128 bytes of bf16)

enum GemmMode : int {
  kGram = 0,       // A = s^2 X X^T (iteration 0) or X X^T, upper tiles, mirrored store
  kPoly = 1,       // B = b A + c A A, upper tiles, mirrored store
  kApply = 2,      // X <- sc (a X + B X): new hi/lo pair
  kApplyLast = 3,  // same, then W <- W decay - lr_scale X and/or O <- X
};

// Kernel variants (GemmParams::staged):
//   kStreamed  128-deep k-blocks in three 64 KB stages; epilogue inputs read into registers,
//              outputs staged in shared memory and written by TMA stores
//   kStaged    64-deep k-blocks; the epilogue's inputs staged in shared memory by TMA.  The
//              Gram and the polynomial store through shared memory by TMA; the applies
//              write their results straight from registers
enum GemmVariant : int { kStreamed = 0, kStaged = 1 };

enum WaitSite : int {
  kSiteProducerEmpty = 1,
  kSiteMmaTmemEmpty = 2,
  kSiteMmaFull = 3,
  kSiteEpilogueFull = 4,
  kSiteTeardownTma = 5,
  kSiteTeardownMma = 6,
  kSiteEpilogueIn = 7,
  kSiteProducerEpi = 8,
};

// One shape class of a wave: `count` matrices of the same rows x cols, stored
// back to back in each scratch buffer.
struct ClassDesc {
  int32_t count;
  int32_t rows, cols;     // stored (row-major) shape
  int32_t m, n;           // m = min(rows, cols): Gram side; n = max
  int32_t tall;           // rows > cols: X is the transpose of the stored matrix
  int32_t ldx;            // row stride of the X buffers (elements, multiple of 8)
  int32_t lda;            // row stride of A and B (elements, multiple of 8)
  int32_t mat_base;       // wave-local index of the class's first matrix
  int32_t tiles_per_mat;
  int32_t tile_begin;     // first flat tile index of this class in the launch
  int32_t mb, nb;         // row / column tile counts of the launch's output
  int32_t ksize;          // reduction length of the launch
  int32_t out_rows, out_cols;
  int32_t a_mn, b_mn;     // operand majorness: 0 = K-major, 1 = MN-major
  int32_t i_fast;         // tile order: row tiles vary fastest
  int64_t x_stride;       // elements between consecutive matrices in the hi buffers
  int64_t lo_stride;      // bytes between consecutive matrices in the lo buffer
  int64_t a_stride;       // elements between consecutive matrices in A / B
  int32_t ldl;            // row stride of the lo buffer (bytes, multiple of 16)
  int32_t pad_;
  __nv_bfloat16* x_hi_cur;   // hi part read this iteration
  __nv_bfloat16* x_hi_next;  // hi part written this iteration
  uint8_t* x_lo;             // lo part (stored 8-bit residual of hi), updated in place
  __nv_bfloat16* a_buf;
  __nv_bfloat16* b_buf;
};

// Per-matrix fields of the final iteration's epilogue.
struct UpdMat {
  void* param;            // W, or nullptr
  float* out;             // O (dense fp32, ld = cols), or nullptr
  int64_t ld_param;
  float lr_scale;         // lr * shape_scale
  int32_t param_bf16;
  int32_t vec_param;      // W rows 16-byte aligned (1: 128-bit accesses) or 32-byte (2: 256-bit)
  int32_t vec_out;        // O rows likewise
};

struct GemmParams {
  CUtensorMap map_a[kMaxClasses];     // operand A of the launch, per class (64 x 128 boxes)
  CUtensorMap map_b[kMaxClasses];     // operand B (64 x 128 boxes)
  CUtensorMap map_out[kMaxClasses];   // epilogue store: Gram -> A, polynomial -> B, apply -> next hi
  CUtensorMap map_out2[kMaxClasses];  // apply: lo (8-bit, 64 x 128 boxes, 64-byte swizzle), load and store
  CUtensorMap map_in[kMaxClasses];    // staged apply: the current hi as epilogue input (64 x 64)
  ClassDesc cls[kMaxClasses];
  int32_t num_classes;
  int32_t total_tiles;
  int32_t staged;                   // GemmVariant of the launch (staged: 64-deep k-blocks,
                                    // MN-major operand maps with 64 x 64 boxes)
  int32_t first_iter;               // iteration 0: s^2 on the Gram, s on the apply
  float a, b, c;                    // this iteration's coefficients
  float decay;                      // 1 - lr * weight_decay (final epilogue)
  const float* scale;               // per wave-local matrix: 1 / (||u|| + eps)
  int32_t* status;                  // device status word (workspace header)
  unsigned long long timeout_ns;
};

struct FinalParams : GemmParams {
  UpdMat upd[kMaxWaveMats];
};

// Elementwise stage: momentum, Nesterov input, bf16 hi/lo split, sum of squares.
struct EwMat {
  const float* g;
  float* m;
  __nv_bfloat16* hi;
  uint8_t* lo;              // stored 8-bit residual of hi, row stride ldl bytes
  int64_t ld_g, ld_m;
  int32_t rows, cols, ldx, ldl;
  int32_t rows_per_chunk;
  int32_t chunk_begin;
  int32_t nchunks;
  int32_t vec;            // 2: 8 per thread, 256-bit; 3: 8 per thread, 128-bit; 1: 4 per thread; 0: scalar
  int32_t index;          // the matrix's index in the caller's descriptor array
};

struct EwParams {
  EwMat mats[kMaxWaveMats];
  int32_t n;
  int32_t total_chunks;
  float beta;
  int32_t nesterov;
  int32_t ns_only;        // read G from `g`, leave momentum alone
  float eps;
  float* partials;        // one fp32 sum of squares per chunk
  float* scale;           // per matrix: 1 / (||u|| + eps)
  float* norm;            // per matrix: ||u||
  int32_t* status;        // workspace header: [0] code, [1] where, [2..3] count of non-finite u (uint64)
};

// Device status codes written into the workspace header (muon_status_t values).
constexpr int kStatusTimeout = 7;
constexpr int kStatusNonfinite = 10;

}  // namespace muon
