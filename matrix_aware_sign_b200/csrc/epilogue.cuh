// epilogue.cuh -- per-stage epilogues of the Newton-Schulz GEMM chain.
//
// Every GEMM kernel (tcgen05 or CUDA-core) hands its accumulator to
// epi_chunk() as NV consecutive columns of one output row. The epilogue
// applies the stage's scalar algebra in float32 and writes the stage's
// outputs. Workspace buffers have leading dims padded to multiples of 128,
// so full vector stores along a row are always in bounds there; user
// buffers are written with bounds checks (and transposed for tall matrices).
#pragma once

#include "kernels.cuh"

namespace smuon {

struct TileCtx {
  const GroupDesc* g;
  const MatDesc* md;
  int32_t stage, iter, last;  // last: this is the final Newton-Schulz step
  int32_t z, Mo, No;
  float s;                    // 1/(||M||_F + eps) of this matrix
  float r;                    // spectral scaling: s r = 1/(||M||_2 + eps); 1 otherwise
  float a, b, c;
  uint32_t flags;
  int32_t bf;                 // operands are bf16 (tcgen05 or SIMT-bf16 mode)
  int32_t split;              // operands are stored as bf16 hi + lo parts
  int32_t sym;                // symmetric m x m stage (Gram, A^2, probe)
  int64_t xlo, mlo;           // element offset of the lo part of an X (m x n) / m x m buffer
  // per-tile copies of the group's and the matrix's pointers and strides: they stay in registers across
  // the epilogue's stores (reading them from the plan after a store would be a dependent load per chunk)
  int64_t ldn, ldm;           // padded leading dims of the group's m x n and m x m buffers
  float* af;                  // f32 A
  void* aop;                  // A operand
  void* bop;                  // B operand
  const float* x_cur;         // B X, steps >= 1: this step's X (plain BF16: f32 master; FP32 mode: the operand)
  const __nv_bfloat16* x_cur_op;  // split mode: this step's X as its hi parts (lo parts xlo further)
  float* xf_next;             // B X: f32 master of the next X (plain BF16 mode only)
  void* xop_next;             // B X: operand of the next X
  const void* m_ptr;          // the user's momentum (the first B X step's source)
  int64_t m_ld;
  void* u_ptr;                // the user's output
  int64_t u_ld;
  int32_t m_dtype, u_dtype, tall, m_vec, u_vec;
  int32_t b_lo;               // write B's lo part: not in a plain leading step, whose B X multiplies hi parts only
  float* xs;                  // this warp's 32 x 33 float transpose buffer in shared memory, or null
};

// The mirrored half of a symmetric stage's 32 x 32 chunk as whole rows: only when the whole warp holds the
// chunk (all 32 rows inside the matrix, all 32 columns valid, the chunk entirely above the diagonal), a test
// that every lane evaluates alike, so no lane of the warp has left early and all take part in the transpose.
__device__ __forceinline__ bool mirror_whole(const TileCtx& t, int row, int col0, int nvalid) {
  const int row_base = row - (int)(threadIdx.x & 31);  // the warp's first row: lane = row within the chunk
  return t.xs != nullptr && nvalid == 32 && row_base + 32 <= t.Mo && col0 >= row_base + 32;
}
// A tall matrix's 32 x 32 chunk read or written as user rows through the warp's transpose buffer: only when
// the whole warp holds it (all 32 wide rows inside the matrix, all 32 wide columns valid), a warp-uniform
// test, so no lane has left early and all take part
__device__ __forceinline__ bool tall_whole(const TileCtx& t, int row, int nvalid) {
  const int row_base = row - (int)(threadIdx.x & 31);
  return t.xs != nullptr && t.tall && nvalid == 32 && row_base + 32 <= t.Mo;
}

// w[r] = the value at (row_base + r, col0 + lane): lane l then holds row col0 + l of the mirrored chunk
__device__ __forceinline__ void xpose32(float* xs, const float* v, float* w) {
  const int lane = threadIdx.x & 31;
  __syncwarp();  // the buffer's previous readers are done
#pragma unroll
  for (int k = 0; k < 32; ++k) xs[lane * 33 + k] = v[k];
  __syncwarp();
#pragma unroll
  for (int r = 0; r < 32; ++r) w[r] = xs[r * 33 + lane];
}

// Gram, A^2 and the probe produce symmetric m x m results. Only tiles that
// reach the diagonal or lie above it are computed; in them an element
// (i, j) is written if j >= i and also mirrored to (j, i) if j > i, so every
// element is written exactly once (deterministically).
__host__ __device__ inline bool sym_stage(int st) {
  return st == ST_GRAM || st == ST_POLY || st == ST_PROBE || st == ST_AA1 || st == ST_AA2;
}

// Tiles are BM x BN with BN = r * BM (r = 1 or 2). Row tm of the tile grid
// holds the column tiles tn >= floor(tm / r); sym_start(tm) counts the tiles
// of the rows before tm, sym_start(T) the tiles of one matrix.
__host__ __device__ inline int sym_start(int tm, int TN, int r) {
  int f;
  if (r == 1) {
    f = tm * (tm - 1) / 2;
  } else {
    const int q = tm / 2;
    f = (tm & 1) ? q * q : q * (q - 1);
  }
  return tm * TN - f;
}

template <int NV>
__device__ __forceinline__ void st_f32_vec(float* p, const float* v) {
#pragma unroll
  for (int q = 0; q < NV / 4; ++q)
    reinterpret_cast<float4*>(p)[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
}

template <int NV>
__device__ __forceinline__ void st_bf16_vec(__nv_bfloat16* p, const float* v) {
  if constexpr (NV % 8 == 0) {
#pragma unroll
    for (int q = 0; q < NV / 8; ++q) {
      uint4 w;
      w.x = pack_bf16x2_rn(v[8 * q + 0], v[8 * q + 1]);
      w.y = pack_bf16x2_rn(v[8 * q + 2], v[8 * q + 3]);
      w.z = pack_bf16x2_rn(v[8 * q + 4], v[8 * q + 5]);
      w.w = pack_bf16x2_rn(v[8 * q + 6], v[8 * q + 7]);
      reinterpret_cast<uint4*>(p)[q] = w;
    }
  } else {
    static_assert(NV % 4 == 0, "chunk must be a multiple of 4");
#pragma unroll
    for (int q = 0; q < NV / 4; ++q) {
      uint2 w;
      w.x = pack_bf16x2_rn(v[4 * q + 0], v[4 * q + 1]);
      w.y = pack_bf16x2_rn(v[4 * q + 2], v[4 * q + 3]);
      reinterpret_cast<uint2*>(p)[q] = w;
    }
  }
}

// Workspace rows (256-byte aligned buffers, leading dims a multiple of 128 elements, chunks starting at a
// multiple of 16 elements) take 256-bit accesses: a lane's 16 floats or 16 bf16 move as whole 32-byte
// sectors, half the L2 requests of 128-bit accesses and no partial-sector writes. User buffers (16-byte
// alignment at most) keep the 128-bit forms above.
__device__ __forceinline__ void st_v8_f32(float* p, const float* v) {
  asm volatile("st.global.v8.f32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};"
               ::"l"(p), "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7])
               : "memory");
}
__device__ __forceinline__ void st_v8_b32(void* p, const uint32_t* w) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};"
               ::"l"(p), "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
               : "memory");
}
__device__ __forceinline__ void ld_v8_f32(const float* p, float* v) {
  asm volatile("ld.global.v8.f32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3]), "=f"(v[4]), "=f"(v[5]), "=f"(v[6]), "=f"(v[7])
               : "l"(p));
}
template <int NV>
__device__ __forceinline__ void st_f32_ws(float* p, const float* v) {
  if constexpr (NV % 8 == 0) {
#pragma unroll
    for (int q = 0; q < NV / 8; ++q) st_v8_f32(p + 8 * q, v + 8 * q);
  } else {
    st_f32_vec<NV>(p, v);
  }
}
template <int NV>
__device__ __forceinline__ void st_bf16_ws(__nv_bfloat16* p, const float* v) {
  if constexpr (NV % 16 == 0) {
#pragma unroll
    for (int q = 0; q < NV / 16; ++q) {
      uint32_t w[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) w[k] = pack_bf16x2_rn(v[16 * q + 2 * k], v[16 * q + 2 * k + 1]);
      st_v8_b32(p + 16 * q, w);
    }
  } else {
    st_bf16_vec<NV>(p, v);
  }
}
template <int NV>
__device__ __forceinline__ void ld_f32_ws(const float* p, float* v) {
  if constexpr (NV % 8 == 0) {
#pragma unroll
    for (int q = 0; q < NV / 8; ++q) ld_v8_f32(p + 8 * q, v + 8 * q);
  } else {
#pragma unroll
    for (int q = 0; q < NV / 4; ++q) {
      float4 t = reinterpret_cast<const float4*>(p)[q];
      v[4 * q] = t.x; v[4 * q + 1] = t.y; v[4 * q + 2] = t.z; v[4 * q + 3] = t.w;
    }
  }
}

// x = hi + lo from the two bf16 parts of a workspace row chunk (split mode's X between steps)
template <int NV>
__device__ __forceinline__ void ld_hilo_ws(const __nv_bfloat16* hi, const __nv_bfloat16* lo, float* x) {
  if constexpr (NV % 16 == 0) {
#pragma unroll
    for (int q = 0; q < NV / 16; ++q) {
      float h[8], l[8];
      ld_v8_f32(reinterpret_cast<const float*>(hi + 16 * q), h);  // 16 bf16 as 8 words
      ld_v8_f32(reinterpret_cast<const float*>(lo + 16 * q), l);
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const uint32_t wh = __float_as_uint(h[k]), wl = __float_as_uint(l[k]);
        x[16 * q + 2 * k] = __uint_as_float(wh << 16) + __uint_as_float(wl << 16);
        x[16 * q + 2 * k + 1] = __uint_as_float(wh & 0xffff0000u) + __uint_as_float(wl & 0xffff0000u);
      }
    }
  } else {
#pragma unroll
    for (int k = 0; k < NV; ++k) x[k] = __bfloat162float(hi[k]) + __bfloat162float(lo[k]);
  }
}

template <int NV>
__device__ __forceinline__ void st_op(void* base, int64_t off, int bf, const float* v) {
  if (bf) st_bf16_ws<NV>(reinterpret_cast<__nv_bfloat16*>(base) + off, v);
  else st_f32_ws<NV>(reinterpret_cast<float*>(base) + off, v);
}

// one operand element (same encodings as st_operand)
__device__ __forceinline__ void st_operand1(const TileCtx& t, void* base, int64_t off, int64_t lo_off, float v,
                                            bool with_lo = true) {
  if (!t.bf) {
    reinterpret_cast<float*>(base)[off] = v;
    return;
  }
  const __nv_bfloat16 hi = __float2bfloat16_rn(v);
  reinterpret_cast<__nv_bfloat16*>(base)[off] = hi;
  if (t.split && with_lo) reinterpret_cast<__nv_bfloat16*>(base)[off + lo_off] = __float2bfloat16_rn(v - __bfloat162float(hi));
}

// operand store: f32, bf16, or bf16 hi at off and lo = bf16(v - hi) at off + lo_off
template <int NV>
__device__ __forceinline__ void st_operand(const TileCtx& t, void* base, int64_t off, int64_t lo_off,
                                           const float* v, bool with_lo = true) {
  if (!t.bf) {
    st_f32_ws<NV>(reinterpret_cast<float*>(base) + off, v);
    return;
  }
  st_bf16_ws<NV>(reinterpret_cast<__nv_bfloat16*>(base) + off, v);
  if (t.split && with_lo) {
    float lo[NV];
#pragma unroll
    for (int k = 0; k < NV; ++k) lo[k] = v[k] - __bfloat162float(__float2bfloat16_rn(v[k]));
    st_bf16_ws<NV>(reinterpret_cast<__nv_bfloat16*>(base) + off + lo_off, lo);
  }
}

template <int NV>
__device__ __forceinline__ void ld_f32_vec(const float* p, float* v) {
#pragma unroll
  for (int q = 0; q < NV / 4; ++q) {
    float4 t = reinterpret_cast<const float4*>(p)[q];
    v[4 * q] = t.x; v[4 * q + 1] = t.y; v[4 * q + 2] = t.z; v[4 * q + 3] = t.w;
  }
}

__device__ __forceinline__ void unpack_bf16x8(const uint4 w, float* o) {
  const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    o[2 * k] = __uint_as_float(u[k] << 16);
    o[2 * k + 1] = __uint_as_float(u[k] & 0xffff0000u);
  }
}

// read a wide-form row chunk (row i, cols j0..j0+NV-1) of a user matrix: a
// wide matrix is read along its row (vector loads when rows are 16-byte
// aligned), a tall one down its column (lanes hold consecutive rows, so each
// warp access is contiguous)
template <int NV>
__device__ __forceinline__ void ld_user(const void* p, int64_t ld, int32_t dtype, int tall, int vec, int row,
                                        int col0, int nvalid, float* out) {
  if (!tall) {
    const int64_t base = (int64_t)row * ld + col0;
    if (vec && nvalid == NV) {
      if (dtype == SMUON_F32) {
        const float* q = reinterpret_cast<const float*>(p) + base;
        if constexpr (NV % 8 == 0) {
          if ((reinterpret_cast<uintptr_t>(q) & 31) == 0) {  // whole 32-byte sectors when the row piece allows
            ld_f32_ws<NV>(q, out);
            return;
          }
        }
        ld_f32_vec<NV>(q, out);
        return;
      }
      if (dtype == SMUON_BF16 && NV % 8 == 0) {
        const uint4* q = reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(p) + base);
#pragma unroll
        for (int k = 0; k < NV / 8; ++k) unpack_bf16x8(q[k], out + 8 * k);
        return;
      }
    }
    if (dtype == SMUON_F32) {
#pragma unroll
      for (int k = 0; k < NV; ++k) out[k] = k < nvalid ? reinterpret_cast<const float*>(p)[base + k] : 0.f;
    } else {
#pragma unroll
      for (int k = 0; k < NV; ++k) out[k] = k < nvalid ? load_as_f32(p, base + k, dtype) : 0.f;
    }
  } else {
    if (dtype == SMUON_F32) {
      const float* q = reinterpret_cast<const float*>(p) + row;
#pragma unroll
      for (int k = 0; k < NV; ++k) out[k] = k < nvalid ? q[(int64_t)(col0 + k) * ld] : 0.f;
    } else {
#pragma unroll
      for (int k = 0; k < NV; ++k) out[k] = k < nvalid ? load_as_f32(p, (int64_t)(col0 + k) * ld + row, dtype) : 0.f;
    }
  }
}

// 1-bit message of a wide-form row chunk (SMUON_BITS output): bit i % 32 of word i / 32 is set iff the
// entry at flat user index i = user_row * cols + user_col is >= 0. cols (= ld) is a multiple of 32.
//  - wide matrix: the lane's NV entries are consecutive user columns of one user row, starting at a
//    multiple of NV: one 32-bit word (NV = 32) or one 16-bit half of a word (NV = 16) per lane.
//  - tall matrix: the wide row is the user column, and the lanes of the warp hold 32 consecutive user
//    columns (row & 31 is the lane) of the same user rows col0 + k: one ballot per k gives the word
//    of user row col0 + k, stored by lane k. Rows and chunk bounds are warp-uniform here because the
//    user's cols (the wide rows) are a multiple of 32, so every lane reaches the ballots.
template <int NV>
__device__ __forceinline__ void st_bits(void* p, int64_t ld, int tall, int row, int col0, int nvalid,
                                        const float* v) {
  if constexpr (NV % 16 == 0) {
    if (!tall) {
      uint32_t bits = 0;
#pragma unroll
      for (int k = 0; k < NV; ++k) bits |= (uint32_t)(v[k] >= 0.f) << k;
      const int64_t e = (int64_t)row * ld + col0;  // a multiple of NV
      if (NV == 32) reinterpret_cast<uint32_t*>(p)[e >> 5] = bits;
      else reinterpret_cast<uint16_t*>(p)[e >> 4] = (uint16_t)bits;
    } else {
      const int lane = threadIdx.x & 31;
      const int64_t row_base = row & ~31;
      uint32_t mine = 0;
#pragma unroll
      for (int k = 0; k < NV; ++k) {
        if (k >= nvalid) break;  // warp-uniform
        const uint32_t b = __ballot_sync(0xffffffffu, v[k] >= 0.f);
        if (lane == k) mine = b;
      }
      if (lane < nvalid) reinterpret_cast<uint32_t*>(p)[((int64_t)(col0 + lane) * ld + row_base) >> 5] = mine;
    }
  }
}

// user-orientation store of a wide-form row chunk (row i, cols j0..j0+NV-1)
template <int NV>
__device__ __forceinline__ void st_user(void* p, int64_t ld, int32_t dtype, int tall, int vec, int row,
                                        int col0, int nvalid, const float* v) {
  if (dtype == SMUON_BITS) {
    st_bits<NV>(p, ld, tall, row, col0, nvalid, v);
    return;
  }
  if (!tall) {
    const int64_t base = (int64_t)row * ld + col0;
    if (vec && nvalid == NV) {
      if (dtype == SMUON_F32) {
        float* q = reinterpret_cast<float*>(p) + base;
        if constexpr (NV % 8 == 0) {
          if ((reinterpret_cast<uintptr_t>(q) & 31) == 0) {
            st_f32_ws<NV>(q, v);
            return;
          }
        }
        st_f32_vec<NV>(q, v);
        return;
      }
      if (dtype == SMUON_I8) {  // the signs only: four entries per 32-bit word
        uint32_t pk[NV / 4];
#pragma unroll
        for (int k = 0; k < NV / 4; ++k)
          pk[k] = (uint32_t)(uint8_t)sign_i8(v[4 * k]) | ((uint32_t)(uint8_t)sign_i8(v[4 * k + 1]) << 8) |
                  ((uint32_t)(uint8_t)sign_i8(v[4 * k + 2]) << 16) | ((uint32_t)(uint8_t)sign_i8(v[4 * k + 3]) << 24);
        uint32_t* q = reinterpret_cast<uint32_t*>(reinterpret_cast<int8_t*>(p) + base);
        if constexpr (NV % 32 == 0) {
          if ((reinterpret_cast<uintptr_t>(q) & 31) == 0) {  // 32 signs as one 32-byte sector
#pragma unroll
            for (int k = 0; k < NV / 32; ++k) st_v8_b32(q + 8 * k, pk + 8 * k);
            return;
          }
        }
        if (NV % 16 == 0) {
#pragma unroll
          for (int k = 0; k < NV / 16; ++k)
            reinterpret_cast<uint4*>(q)[k] = make_uint4(pk[4 * k], pk[4 * k + 1], pk[4 * k + 2], pk[4 * k + 3]);
        } else {
#pragma unroll
          for (int k = 0; k < NV / 4; ++k) q[k] = pk[k];
        }
        return;
      }
      __nv_bfloat16* qb = reinterpret_cast<__nv_bfloat16*>(p) + base;
      if constexpr (NV % 16 == 0) {
        if ((reinterpret_cast<uintptr_t>(qb) & 31) == 0) {
          st_bf16_ws<NV>(qb, v);
          return;
        }
      }
      st_bf16_vec<NV>(qb, v);
      return;
    }
#pragma unroll
    for (int q = 0; q < NV; ++q)
      if (q < nvalid) store_from_f32(p, base + q, dtype, v[q]);
  } else if (dtype == SMUON_BF16) {
    __nv_bfloat16* q = reinterpret_cast<__nv_bfloat16*>(p) + row;
#pragma unroll
    for (int k = 0; k < NV; ++k)
      if (k < nvalid) q[(int64_t)(col0 + k) * ld] = __float2bfloat16_rn(v[k]);
  } else if (dtype == SMUON_I8) {
    int8_t* q = reinterpret_cast<int8_t*>(p) + row;
#pragma unroll
    for (int k = 0; k < NV; ++k)
      if (k < nvalid) q[(int64_t)(col0 + k) * ld] = sign_i8(v[k]);
  } else {
    float* q = reinterpret_cast<float*>(p) + row;
#pragma unroll
    for (int k = 0; k < NV; ++k)
      if (k < nvalid) q[(int64_t)(col0 + k) * ld] = v[k];
  }
}

// symmetric-stage stores of a row chunk: elements k >= ds are written in
// place (vector store when the whole chunk is, the row being padded), and
// elements k >= ms (strictly above the diagonal) are also written transposed;
// lanes hold consecutive rows, so each transposed store of a warp is contiguous
template <int NV>
__device__ __forceinline__ void sym_store_f32(const TileCtx& t, float* base, int row, int col0, int nvalid,
                                              int ds, int ms, const float* v) {
  const int64_t m = t.Mo, ld = t.ldm;
  const int64_t off = ((int64_t)t.z * m + row) * ld + col0;
  if (ds == 0) {
    st_f32_ws<NV>(base + off, v);
  } else {
#pragma unroll
    for (int k = 0; k < NV; ++k)
      if (k >= ds && k < nvalid) base[off + k] = v[k];
  }
  if (!t.sym) return;
  if constexpr (NV == 32) {
    if (mirror_whole(t, row, col0, nvalid)) {
      float w[32];
      xpose32(t.xs, v, w);
      const int lane = threadIdx.x & 31;
      st_f32_ws<32>(base + ((int64_t)t.z * m + col0 + lane) * ld + (row - lane), w);
      return;
    }
  }
#pragma unroll
  for (int k = 0; k < NV; ++k)
    if (k >= ms && k < nvalid) base[((int64_t)t.z * m + col0 + k) * ld + row] = v[k];
}

template <int NV>
__device__ __forceinline__ void sym_store_operand(const TileCtx& t, void* base, int row, int col0, int nvalid,
                                                  int ds, int ms, const float* v, bool with_lo = true) {
  const int64_t m = t.Mo, ld = t.ldm;
  const int64_t off = ((int64_t)t.z * m + row) * ld + col0;
  if (ds == 0) {
    st_operand<NV>(t, base, off, t.mlo, v, with_lo);
  } else {
#pragma unroll
    for (int k = 0; k < NV; ++k)
      if (k >= ds && k < nvalid) st_operand1(t, base, off + k, t.mlo, v[k], with_lo);
  }
  if (!t.sym) return;
  if constexpr (NV == 32) {
    if (mirror_whole(t, row, col0, nvalid)) {
      float w[32];
      xpose32(t.xs, v, w);
      const int lane = threadIdx.x & 31;
      st_operand<32>(t, base, ((int64_t)t.z * m + col0 + lane) * ld + (row - lane), t.mlo, w, with_lo);
      return;
    }
  }
#pragma unroll
  for (int k = 0; k < NV; ++k)
    if (k >= ms && k < nvalid) st_operand1(t, base, ((int64_t)t.z * m + col0 + k) * ld + row, t.mlo, v[k], with_lo);
}

// largest tm with sym_start(tm) <= r (binary search), then the column tile
__device__ __forceinline__ void sym_decode(int r, int T, int TN, int ratio, int& tm, int& tn) {
  int lo = 0, hi = T - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (sym_start(mid, TN, ratio) <= r) lo = mid; else hi = mid - 1;
  }
  tm = lo;
  tn = lo / ratio + (r - sym_start(lo, TN, ratio));
}

// first cached transform Q_1 = aI + B_0 (CacheMuon fresh solve, reading R14);
// symmetric like B_0, stored with the same triangle rule
template <int NV>
__device__ __forceinline__ void emit_q1(const TileCtx& t, int row, int col0, int nvalid, int ds, int ms,
                                        const float* B) {
  float q[NV];
#pragma unroll
  for (int k = 0; k < NV; ++k) q[k] = B[k] + ((row == col0 + k) ? t.a : 0.f);
  if (t.iter == t.last) {  // K == 1: Q_1 is the final transform, in the user's bf16 buffer
    __nv_bfloat16* Q = reinterpret_cast<__nv_bfloat16*>(t.md->q_ptr);
    const int64_t ld = t.md->q_ld;
#pragma unroll
    for (int k = 0; k < NV; ++k) {
      if (k >= ds && k < nvalid) Q[(int64_t)row * ld + col0 + k] = __float2bfloat16_rn(q[k]);
      if (k >= ms && k < nvalid) Q[(int64_t)(col0 + k) * ld + row] = __float2bfloat16_rn(q[k]);
    }
  }
  if (t.iter != t.last || (t.flags & SMUON_NS_GRAM_ONLY)) {  // the Gram-only solve also multiplies by it
    if (t.bf) sym_store_f32<NV>(t, t.g->qf[1], row, col0, nvalid, ds, ms, q);
    sym_store_operand<NV>(t, t.g->qop[1], row, col0, nvalid, ds, ms, q);
  }
}

// v[] holds the raw accumulator of D = A_op * B_op at (row, col0..col0+NV-1). kStage is the stage when
// the caller knows it at compile time (then only that stage's code and context stay live), else -1.
template <int NV, int kStage = -1>
__device__ __forceinline__ void epi_chunk(const TileCtx& t, int row, int col0, float* v,
                                          float* probe_acc) {
  if (row >= t.Mo || col0 >= t.No) return;
  const int nvalid = min(NV, t.No - col0);
  const GroupDesc& g = *t.g;
  const int m = t.Mo;
  // symmetric stages: elements k >= ds are on or above the diagonal, k >= ms strictly above
  const int ds = t.sym ? max(0, row - col0) : 0;
  const int ms = t.sym ? max(0, row - col0 + 1) : NV;
  switch (kStage >= 0 ? kStage : t.stage) {
    case ST_GRAM: {
      if (ds >= nvalid) break;  // the chunk lies below the diagonal
      const float sc = (t.iter == 0 && !(t.flags & SMUON_NS_NO_NORMALIZE)) ? t.s * t.s : 1.f;
      if (t.c != 0.f) {
#pragma unroll
        for (int k = 0; k < NV; ++k) v[k] *= sc;
        if (t.af) sym_store_f32<NV>(t, t.af, row, col0, nvalid, ds, ms, v);  // split mode: A's hi + lo serve
        if (t.bf) sym_store_operand<NV>(t, t.aop, row, col0, nvalid, ds, ms, v);
      } else {
        if (t.flags & SMUON_NS_SPECTRAL) {  // f32 A_0 for the largest-eigenvalue estimate
          float a0[NV];
#pragma unroll
          for (int k = 0; k < NV; ++k) a0[k] = sc * v[k];
          sym_store_f32<NV>(t, t.af, row, col0, nvalid, ds, ms, a0);
        }
#pragma unroll
        for (int k = 0; k < NV; ++k) v[k] = t.b * (sc * v[k]);
        sym_store_operand<NV>(t, t.bop, row, col0, nvalid, ds, ms, v, t.b_lo);
        if ((t.flags & SMUON_NS_EMIT_Q) && t.iter == 0) emit_q1<NV>(t, row, col0, nvalid, ds, ms, v);
      }
      break;
    }
    case ST_POLY: {
      if (ds >= nvalid) break;
      const int64_t off = ((int64_t)t.z * m + row) * t.ldm + col0;
      float A[NV];
      if (t.af) {
        ld_f32_ws<NV>(t.af + off, A);
      } else {  // split mode: A = hi + lo
        const __nv_bfloat16* ah = reinterpret_cast<const __nv_bfloat16*>(t.aop);
        ld_hilo_ws<NV>(ah + off, ah + off + t.mlo, A);
      }
      // spectral scaling at the first step: A' = r^2 A, so B = b r^2 A + c r^4 A^2 (r = 1 otherwise)
      const float r2 = t.iter == 0 ? t.r * t.r : 1.f;
#pragma unroll
      for (int k = 0; k < NV; ++k) v[k] = t.b * (r2 * A[k]) + t.c * ((r2 * r2) * v[k]);
      sym_store_operand<NV>(t, t.bop, row, col0, nvalid, ds, ms, v, t.b_lo);
      if ((t.flags & SMUON_NS_EMIT_Q) && t.iter == 0) emit_q1<NV>(t, row, col0, nvalid, ds, ms, v);
      break;
    }
    case ST_AXPY: {
      const bool first = (t.iter == 0);
      // s r: the Frobenius scale, times r for spectral scaling; with c = 0 the first B = b A was
      // written before r was known, so its product takes the r^2 of A' = r^2 A here
      const float sc = (first && !(t.flags & SMUON_NS_NO_NORMALIZE)) ? t.s * t.r : 1.f;
      const float sv = (first && t.c == 0.f) ? sc * (t.r * t.r) : sc;
      const int64_t off = ((int64_t)t.z * m + row) * t.ldn + col0;
      float x[NV];
      bool whole_tall = false;
      if constexpr (NV == 32) whole_tall = tall_whole(t, row, nvalid);
      if (first && t.bf && whole_tall && t.m_dtype == SMUON_F32) {
        // X_0 from a tall f32 momentum: lane l reads user row col0 + l (the wide rows row_base.. as 32
        // contiguous floats), then the transpose gives each lane its wide row
        if constexpr (NV == 32) {
          const int lane = threadIdx.x & 31;
          const float* urow = reinterpret_cast<const float*>(t.m_ptr) + (int64_t)(col0 + lane) * t.m_ld + (row - lane);
          float y[32];
          if (t.m_vec) ld_f32_vec<32>(urow, y);
          else
#pragma unroll
            for (int k = 0; k < 32; ++k) y[k] = urow[k];
          xpose32(t.xs, y, x);
        }
      } else if (first && t.bf) {
        // X_0 read from the user's momentum in its own dtype and orientation
        ld_user<NV>(t.m_ptr, t.m_ld, t.m_dtype, t.tall, t.m_vec, row, col0, nvalid, x);
      } else if (t.split) {
        ld_hilo_ws<NV>(t.x_cur_op + off, t.x_cur_op + off + t.xlo, x);
      } else {
        ld_f32_ws<NV>(t.x_cur + off, x);
      }
#pragma unroll
      for (int k = 0; k < NV; ++k) x[k] = t.a * (sc * x[k]) + sv * v[k];
      if (t.iter != t.last) {
        if (t.bf && !t.split) st_f32_ws<NV>(t.xf_next + off, x);
        st_operand<NV>(t, t.xop_next, off, t.xlo, x);
      } else if (whole_tall && t.u_dtype != SMUON_BITS) {
        // U of a tall matrix: the transpose gives lane l user row col0 + l, written as 32 contiguous entries
        if constexpr (NV == 32) {
          const int lane = threadIdx.x & 31;
          float y[32];
          xpose32(t.xs, x, y);
          st_user<32>(t.u_ptr, t.u_ld, t.u_dtype, 0, t.u_vec, col0 + lane, row - lane, 32, y);
        }
      } else {
        st_user<NV>(t.u_ptr, t.u_ld, t.u_dtype, t.tall, t.u_vec, row, col0, nvalid, x);
      }
      break;
    }
    case ST_QAXPY: {
      const int64_t off = ((int64_t)t.z * m + row) * t.ldm + col0;
      float q[NV];
      const float* src = t.bf ? g.qf[t.iter & 1] : reinterpret_cast<const float*>(g.qop[t.iter & 1]);
      ld_f32_ws<NV>(src + off, q);
#pragma unroll
      for (int k = 0; k < NV; ++k) q[k] = t.a * q[k] + v[k];
      if (t.iter == t.last)
        st_user<NV>(t.md->q_ptr, t.md->q_ld, SMUON_BF16, 0, (t.md->vec >> 2) & 1, row, col0, nvalid, q);
      if (t.iter != t.last || (t.flags & SMUON_NS_GRAM_ONLY)) {  // Q_K X_0 reads the workspace copy
        const int nb = (t.iter + 1) & 1;
        if (t.bf) st_f32_ws<NV>(g.qf[nb] + off, q);
        st_operand<NV>(t, g.qop[nb], off, t.mlo, q);
      }
      break;
    }
    case ST_QX: {  // Gram-only fresh solve: U = s Q_K X_0
#pragma unroll
      for (int k = 0; k < NV; ++k) v[k] *= t.s;
      st_user<NV>(t.u_ptr, t.u_ld, t.u_dtype, t.tall, t.u_vec, row, col0, nvalid, v);
      break;
    }
    case ST_REUSE: {
      const int64_t off = ((int64_t)t.z * m + row) * t.ldn + col0;
#pragma unroll
      for (int k = 0; k < NV; ++k) v[k] *= t.s;
      st_user<NV>(t.u_ptr, t.u_ld, t.u_dtype, t.tall, t.u_vec, row, col0, nvalid, v);
      if (!(t.flags & SMUON_NS_GRAM_ONLY)) st_op<NV>(g.xop[1], off, t.bf, v);  // the probe's operand
      break;
    }
    case ST_AA1:
    case ST_AA2: {
      // Gram-only fresh solve: Y' = a Y + B Y with Y = A_k (first) or T = P_k A_k
      // (second); both are symmetric (polynomials in A_k), stored by the triangle rule
      if (ds >= nvalid) break;
      const bool first = t.stage == ST_AA1;
      const int64_t off = ((int64_t)t.z * m + row) * t.ldm + col0;
      float y[NV];
      ld_f32_ws<NV>((first ? g.af : g.af2) + off, y);
#pragma unroll
      for (int k = 0; k < NV; ++k) v[k] = t.a * y[k] + v[k];
      sym_store_f32<NV>(t, first ? g.af2 : g.af, row, col0, nvalid, ds, ms, v);
      sym_store_operand<NV>(t, first ? g.aop2 : g.aop, row, col0, nvalid, ds, ms, v);
      break;
    }
    case ST_PROBE: {
      float acc = 0.f;
#pragma unroll
      for (int k = 0; k < NV; ++k) {
        if (k >= ds && k < nvalid) {
          const float r = v[k] - ((row == col0 + k) ? 1.f : 0.f);
          acc = fmaf(k >= ms ? 2.f * r : r, r, acc);  // an element above the diagonal stands for its mirror too
        }
      }
      *probe_acc += acc;
      break;
    }
    default: break;
  }
}

// B X epilogue with its X source already read (x[]): X' = a s X + s B X (first
// step) or a X + B X, written as the next step's operand (and, in plain BF16, its f32 master), or
// into the user's U after the last step
template <int NV>
__device__ __forceinline__ void epi_axpy_src(const TileCtx& t, int row, int col0, const float* v, float* x) {
  if (row >= t.Mo || col0 >= t.No) return;
  const int nvalid = min(NV, t.No - col0);
  const float sc = (t.iter == 0 && !(t.flags & SMUON_NS_NO_NORMALIZE)) ? t.s * t.r : 1.f;
  const float sv = (t.iter == 0 && t.c == 0.f) ? sc * (t.r * t.r) : sc;
#pragma unroll
  for (int k = 0; k < NV; ++k) x[k] = t.a * (sc * x[k]) + sv * v[k];
  if (t.iter != t.last) {
    const int64_t off = ((int64_t)t.z * t.Mo + row) * t.ldn + col0;
    if (!t.split) st_f32_ws<NV>(t.xf_next + off, x);  // split mode: hi + lo is the next step's source
    st_operand<NV>(t, t.xop_next, off, t.xlo, x);
  } else {
    st_user<NV>(t.u_ptr, t.u_ld, t.u_dtype, t.tall, t.u_vec, row, col0, nvalid, x);
  }
}

// per-tile context from a linear tile index of stage st
__device__ __forceinline__ TileCtx make_ctx(const PlanHeader& h, int st, int iter, int tile,
                                            int& tm, int& tn) {
  TileCtx t;
  const int gi = find_group(h, st, tile);
  const GroupDesc& g = h.groups[gi];
  const int local = tile - g.tile_begin[st];
  if (sym_stage(st)) {
    const int T = g.tiles_m[st], TN = g.tiles_n[st], ratio = h.sym_ratio[st];
    const int per = sym_start(T, TN, ratio);
    t.z = local / per;
    sym_decode(local - t.z * per, T, TN, ratio, tm, tn);
  } else {
    // column-major within a matrix: consecutive tiles share the right-hand
    // operand's column panel (X or Q), which then stays in L2
    const int per = g.tiles_m[st] * g.tiles_n[st];
    t.z = local / per;
    const int rem = local - t.z * per;
    tn = rem / g.tiles_m[st];
    tm = rem - tn * g.tiles_m[st];
  }
  t.sym = sym_stage(st) ? 1 : 0;
  t.g = &h.groups[gi];
  t.md = &h.mats[g.first_mat + t.z];
  t.stage = st;
  t.iter = iter;
  t.last = h.iters - 1;
  t.Mo = g.m;
  t.No = wide_out_stage(st) ? g.n : g.m;
  t.s = h.scale[g.first_mat + t.z];
  t.r = (h.flags & SMUON_NS_SPECTRAL) ? h.rscale[g.first_mat + t.z] : 1.f;
  t.a = h.a; t.b = h.b; t.c = h.c;
  t.flags = h.flags;
  t.bf = (h.mode != MODE_SIMT_F32);
  t.split = (h.flags & SMUON_NS_SPLIT_BF16) ? 1 : 0;
  t.xlo = (int64_t)g.count * g.m * g.ldn;
  t.mlo = (int64_t)g.count * g.m * g.ldm;
  t.ldn = g.ldn;
  t.ldm = g.ldm;
  t.af = g.af;
  t.aop = g.aop;
  t.bop = g.bop;
  t.x_cur = t.bf ? g.xf[iter & 1] : reinterpret_cast<const float*>(g.xop[iter & 1]);
  t.x_cur_op = reinterpret_cast<const __nv_bfloat16*>(g.xop[iter & 1]);
  t.xf_next = g.xf[(iter + 1) & 1];
  t.xop_next = g.xop[(iter + 1) & 1];
  const MatDesc& md = *t.md;
  t.m_ptr = md.m_ptr;
  t.m_ld = md.m_ld;
  t.u_ptr = md.u_ptr;
  t.u_ld = md.u_ld;
  t.m_dtype = md.m_dtype;
  t.u_dtype = md.u_dtype;
  t.tall = md.tall;
  t.m_vec = md.vec & 1;
  t.u_vec = (md.vec >> 1) & 1;
  t.b_lo = !plain_lead_stage(h.flags, ST_AXPY, iter, g.m);
  t.xs = nullptr;
  return t;
}

}  // namespace smuon
