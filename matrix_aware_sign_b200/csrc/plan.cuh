// plan.cuh -- device-resident description of one batched Newton-Schulz call.
//
// The host builds a Plan (groups of same-shape matrices, per-matrix user
// pointers, workspace buffers, TMA tensor maps and per-stage tile tables),
// uploads it into the head of the caller's workspace with a kernel whose
// parameters carry the bytes (no host->device memcpy, so a call can be
// captured in a CUDA graph), and every kernel of the call reads it from there.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "smuon.h"

namespace smuon {

constexpr int kMaxWorkers = 64;
constexpr int kMaxSchedCtas = 1024;  // most CTAs a tensor-core stage is scheduled over
constexpr int kShallowMaxK = 1024;    // stages with K up to this use the shallow smem ring

// Stages of the Newton-Schulz chain. Each is one grouped GEMM launch
// D = A_op * B_op over every matrix of the batch, with its own epilogue.
enum Stage : int32_t {
  ST_GRAM = 0,   // A = s^2 X X^T                      (m x m, K = n)
  ST_POLY = 1,   // B = b A + c A^2                      (m x m, K = m)
  ST_AXPY = 2,   // X' = a s X + s B X                   (m x n, K = m)
  ST_QAXPY = 3,  // Q' = a Q + B Q                       (m x m, K = m)
  ST_REUSE = 4,  // D_hat = s Q X_t                      (m x n, K = m)
  ST_PROBE = 5,  // sum (D_hat D_hat^T - I)^2 per tile   (m x m, K = n)
  ST_AA1 = 6,    // T = a A + B A = P A                  (m x m, K = m)  Gram-only fresh solve
  ST_AA2 = 7,    // A' = a T + B T = P^2 A               (m x m, K = m)  Gram-only fresh solve
  ST_QX = 8,     // U = s Q_K X_0                        (m x n, K = m)  Gram-only fresh solve
  ST_COUNT = 9
};

// stages whose output is the m x n wide form (the others are m x m)
__host__ __device__ inline bool wide_out_stage(int st) { return st == ST_AXPY || st == ST_REUSE || st == ST_QX; }

// stages whose operands carry hi and lo parts in split mode (all but the
// CacheMuon reuse and probe products, which read the cached bf16 transform)
__host__ __device__ inline bool split_stage(int st) { return st != ST_REUSE && st != ST_PROBE; }

// split mode with SMUON_NS_PLAIN_LEAD(k): the Newton-Schulz steps iter < k of a matrix group multiply only
// the hi parts of their operands (one MMA per product; the lo parts are still written for the later
// steps): every group's first step, and the later ones only where the smaller side m is at least
// kPlainLeadMinM (below that the normalised singular values start near 1/sqrt(m), too large for a second
// plain step)
constexpr int kPlainLeadMinM = 512;
__host__ __device__ inline bool plain_lead_stage(uint32_t flags, int st, int iter, int m) {
  return iter < (int)((flags >> 12) & 7u) && (iter == 0 || m >= kPlainLeadMinM) &&
         (st == ST_GRAM || st == ST_POLY || st == ST_AXPY);
}

enum Mode : int32_t { MODE_TC_BF16 = 0, MODE_SIMT_F32 = 1, MODE_SIMT_BF16 = 2 };

// Tile-list entries of the tensor-core stages: a tile id, or (B X stage only) half of a tile, the left or the
// right half of its columns, flagged by bit 30 with the side in bit 29. The last partial wave of a B X stage
// is split into half tiles when at most half the lists would take one (the wave then ends in half the time).
constexpr int32_t kHalfTileFlag = 1 << 30;
constexpr int32_t kHalfTileSide = 1 << 29;
__host__ __device__ inline bool half_tile_stage(int st) { return st == ST_AXPY; }

// one user matrix (user orientation rows x cols); NS runs on the wide form
// m x n with m = min(rows, cols): a tall matrix is read transposed.
struct MatDesc {
  void* m_ptr;      // momentum / input matrix
  int64_t m_ld;
  const void* g_ptr;  // gradient, nullable
  int64_t g_ld;
  void* u_ptr;      // polar-factor output (or D_hat for the probe)
  int64_t u_ld;
  void* q_ptr;      // bf16 m x m cached transform (EMIT_Q output, or REUSE input)
  int64_t q_ld;
  int32_t m_dtype, g_dtype, u_dtype;
  int32_t vec;            // bit 0: M rows 16-byte aligned (vector reads); bit 1: U rows; bit 2: Q rows;
                          // bit 3: M and G suit the vectorised momentum tile
  int32_t rows, cols, tall, group;
  int32_t z;              // index of this matrix inside its group
  int32_t mom_begin;      // first momentum tile (= partial-sum slot)
  int32_t mom_tiles_c;    // 64x64 tiles along cols (user orientation)
  int32_t mom_count;      // number of momentum tiles
  int32_t tm_src;         // f32 map of M for the first B X epilogue's source (-1: none)
  int32_t pad0;
  int64_t lz_off;         // spectral scaling: this matrix's Lanczos vectors in PlanHeader::lz
};

// matrices of one wide shape m x n, stored contiguously in the workspace
struct GroupDesc {
  int32_t m, n, count, first_mat;
  int64_t ldn, ldm;       // padded leading dims (elements), multiples of 128
  void* xop[2];           // X operand [count][m][ldn] (bf16, or f32 in FP32 mode)
  float* xf[2];           // f32 master of X for iterations >= 1 (plain BF16 mode; split mode keeps hi + lo)
  float* af;              // f32 A [count][m][ldm]
  void* aop;              // A operand (bf16 modes; == af in FP32 mode)
  void* bop;              // B operand [count][m][ldm]
  float* qf[2];           // f32 master of Q (EMIT_Q)
  void* qop[2];           // Q operand
  float* af2;             // Gram-only fresh solve: f32 T = P A between the two A updates
  void* aop2;             // T operand
  int32_t tm_x_k[2];      // tensor-map indices: X K-major box {64,128}
  int32_t tm_x_mn[2];     // X MN-major box {64,64}
  int32_t tm_a_k, tm_b_k; // A / B K-major box {64,128}
  int32_t tm_q_mn[2];     // Q MN-major box {64,64}
  int32_t tm_uq_k;        // user Q K-major (REUSE A operand)
  int32_t tm_a_kw;        // A K-major box {64,256} (B operand of 256-wide tiles)
  int32_t tm_x_kw[2];     // X K-major box {64,256}
  int32_t tm_t_k, tm_t_kw; // T K-major boxes {64,128} and {64,256}
  int32_t tm_q_k[2];      // Q K-major box {64,128} (left operand of Q_K X_0)
  int32_t tm_xf[2];       // B X epilogue source of X_i for steps >= 1: the f32 master, box {32,128}, 128B
                          // swizzle (plain BF16), or the bf16 hi and lo parts, box {32,128}, 64B swizzle (split)
  int32_t tiles_m[ST_COUNT], tiles_n[ST_COUNT], tile_begin[ST_COUNT];
};

struct PlanHeader {
  int32_t n_mats, n_groups, n_tmaps, mode;
  int32_t iters;
  uint32_t flags;
  float a, b, c, eps;
  float beta;
  float gamma;              // probe threshold
  int32_t total_mom_tiles;
  int32_t tile_bm, tile_bn; // tile shape of the GEMM kernel the tables are built for (256 x 256 for SM pairs)
  int32_t pair;             // tensor-core stages on SM pairs (clusters of two CTAs, one 256 x 256 tile each)
  int32_t pad_pair;
  int32_t total_tiles[ST_COUNT];
  int32_t sym_ratio[ST_COUNT];  // BN / BM of the symmetric stages' tiles (1 or 2)
  float* partials;          // [total_mom_tiles][8] sum of squares per momentum tile and warp
  float* scale;             // [n_mats] s = 1/(||M||_F + eps)
  float* probe_partials;    // [total PROBE tiles]
  const int32_t* mom_begin; // [n_mats + 1] first momentum tile of each matrix (compact, for the tile search)
  // tensor-core stages: each CTA walks its own list of tiles, balanced on the
  // host by tile cost (longest first onto the least loaded CTA)
  const int32_t* sched;             // tile ids of every stage, CTA after CTA
  const int32_t* sched_begin;       // per stage: first list entry of each CTA (sched_ctas + 1 entries)
  int32_t sched_off[ST_COUNT];      // offset of each stage's tile ids in sched
  int32_t sched_boff[ST_COUNT];     // offset of each stage's begin array in sched_begin
  int32_t sched_ctas[ST_COUNT];     // CTAs of each stage's launch
  int32_t max_k[ST_COUNT];          // longest K of each stage over the groups (picks the smem ring depth)
  int32_t axpy_tma;                 // the B X epilogue's X source is staged in shared memory by TMA
  int32_t starve_tc;                // failure-detection test: the tensor-core stages' producers issue nothing
  uint64_t wait_cycles;             // budget of one pipeline wait in the tensor-core stages (SM clocks)
  float* rscale;                    // spectral scaling: r per matrix (X_0 = s r M), or null
  float* lz;                        // Lanczos vectors of every matrix (kLanczosSteps + 2 vectors of m each)
  float* lz_ab;                     // [n_mats][2 kLanczosSteps] Lanczos alpha, beta
  const int32_t* lz_rows;           // [n_mats + 1] first row of each matrix in the flattened row range
  int32_t* lz_act;                  // matrices still iterating: [count][rows prefix, n_mats + 1][matrix, n_mats]
  GroupDesc* groups;        // device pointers into the plan region
  MatDesc* mats;
  CUtensorMap* tmaps;
  int32_t* status;          // nullable
  float* d_err;             // probe outputs
  int32_t* d_accept;
  cachemuon_counters* counters;
};

struct Plan {
  PlanHeader h;
};

// ---------------------------------------------------------------- helpers
__host__ __device__ inline int64_t round_up(int64_t x, int64_t m) { return (x + m - 1) / m * m; }
__host__ __device__ inline int32_t ceil_div(int64_t x, int64_t m) { return (int32_t)((x + m - 1) / m); }

__device__ inline float load_as_f32(const void* p, int64_t idx, int32_t dtype) {
  if (dtype == SMUON_F32) return reinterpret_cast<const float*>(p)[idx];
  if (dtype == SMUON_BF16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p)[idx]);
  return (float)reinterpret_cast<const int8_t*>(p)[idx];
}

// an I8 destination receives the entrywise sign: +1 for v >= 0 (-0 included), -1 otherwise (NaN included)
__device__ inline int8_t sign_i8(float v) { return v >= 0.f ? (int8_t)1 : (int8_t)-1; }

__device__ inline void store_from_f32(void* p, int64_t idx, int32_t dtype, float v) {
  if (dtype == SMUON_F32) reinterpret_cast<float*>(p)[idx] = v;
  else if (dtype == SMUON_I8) reinterpret_cast<int8_t*>(p)[idx] = sign_i8(v);
  else reinterpret_cast<__nv_bfloat16*>(p)[idx] = __float2bfloat16_rn(v);
}

// locate the group of a linear tile index of stage st (groups are few: linear scan)
__device__ inline int find_group(const PlanHeader& h, int st, int tile) {
  int g = 0;
  while (g + 1 < h.n_groups && h.groups[g + 1].tile_begin[st] <= tile) ++g;
  return g;
}

// locate the matrix owning a momentum tile (binary search over a compact
// array of first tiles, which stays in L1 across the tiles of a CTA)
__device__ inline int find_mat_by_mom_tile(const PlanHeader& h, int tile) {
  const int32_t* __restrict__ b = h.mom_begin;
  int lo = 0, hi = h.n_mats - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (__ldg(b + mid) <= tile) lo = mid; else hi = mid - 1;
  }
  return lo;
}

}  // namespace smuon
