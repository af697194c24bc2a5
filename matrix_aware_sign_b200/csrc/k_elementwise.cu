// k_elementwise.cu -- bandwidth-bound kernels of the optimizer step.
//
//  * k_plan_upload     copies a Plan (carried in kernel parameters) into the workspace
//  * k_momentum        M <- beta*M + G, per-tile sum of squares, X0 in wide form
//  * k_norm_finalize   s = 1/(||M||_F + eps) per matrix (deterministic order)
//  * k_vote_update     fused sign / pack / popcount (or int8) vote / W update
//  * k_sign_pack       signs and 1-bit packing only
//  * k_vote            vote from packed bits or int8 signs
//  * k_update_src      W update from a vote matrix or a dense direction
//  * k_lion_sign       LionMuon sign step (G_hat, vote, W and EMA update)
//  * k_lion_mean       LionMuon Muon-step prologue (mean of G_hat, EMA update)
//  * k_probe_finalize  CacheMuon residual, accept flag and counters
//  * k_harness_gaussian  counter-based gradient streams written out (harness)
#include <algorithm>

#include "counter_rng.cuh"
#include "kernels.cuh"

namespace smuon {

// --------------------------------------------------------------------------
__global__ void k_plan_upload(const __grid_constant__ UploadChunk c) {
  const int n16 = c.bytes / 16;
  const uint4* src = reinterpret_cast<const uint4*>(c.data);
  uint4* dst = reinterpret_cast<uint4*>(c.dst);
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n16; i += gridDim.x * blockDim.x)
    dst[i] = src[i];
}

// X0 operand element: f32, bf16, or bf16 hi + lo (lo part count*m*ldn elements later)
__device__ __forceinline__ void put_x0(const GroupDesc& g, int bf, int split, int64_t o, float v) {
  if (!bf) {
    reinterpret_cast<float*>(g.xop[0])[o] = v;
    return;
  }
  const __nv_bfloat16 hi = __float2bfloat16_rn(v);
  reinterpret_cast<__nv_bfloat16*>(g.xop[0])[o] = hi;
  if (split)
    reinterpret_cast<__nv_bfloat16*>(g.xop[0])[o + (int64_t)g.count * g.m * g.ldn] =
        __float2bfloat16_rn(v - __bfloat162float(hi));
}

// --------------------------------------------------------------------------
// SignMuon summary, algorithm flow step 1: momentum update (reading R1) fused
// with the sum of squares for the Frobenius norm and the bf16/f32 operand
// copy of X0 in the wide orientation (tall matrices transposed through smem).
__device__ __forceinline__ void put_x0_4(const GroupDesc& g, int bf, int split, int64_t o, const float* v) {
  if (!bf) {
    *reinterpret_cast<float4*>(reinterpret_cast<float*>(g.xop[0]) + o) = make_float4(v[0], v[1], v[2], v[3]);
    return;
  }
  uint2 hi;
  hi.x = pack_bf16x2_rn(v[0], v[1]);
  hi.y = pack_bf16x2_rn(v[2], v[3]);
  *reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(g.xop[0]) + o) = hi;
  if (split) {
    float lo[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) lo[k] = v[k] - __bfloat162float(__float2bfloat16_rn(v[k]));
    uint2 l;
    l.x = pack_bf16x2_rn(lo[0], lo[1]);
    l.y = pack_bf16x2_rn(lo[2], lo[3]);
    *reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(g.xop[0]) + o + (int64_t)g.count * g.m * g.ldn) = l;
  }
}

// four CTAs per SM (at most 64 registers): the tile loop waits on its loads, so more warps in flight
// move more bytes (measured 77% -> 86% of HBM on the ResNet-50 set)
__global__ void __launch_bounds__(256, 4) k_momentum(const Plan* plan, const int32_t* skip) {
  if (skip && *skip) return;
  const PlanHeader& h = plan->h;
  __shared__ float tile[64][65];  // the transpose of a tall matrix's tile
  const int bf = (h.mode != MODE_SIMT_F32);
  const int split = (h.flags & SMUON_NS_SPLIT_BF16) != 0;
  const int total = h.total_mom_tiles;
  float* __restrict__ partials = h.partials;
  for (int t = blockIdx.x; t < total; t += gridDim.x) {
    const int mi = find_mat_by_mom_tile(h, t);
    // descriptor fields live in registers: the stores below may not be assumed
    // to leave global descriptors untouched, so nothing is re-read after them
    const MatDesc md = h.mats[mi];
    GroupDesc g;
    {
      const GroupDesc& gg = h.groups[md.group];
      g.m = gg.m; g.count = gg.count; g.ldn = gg.ldn; g.xop[0] = gg.xop[0];
    }
    const float beta = h.beta;
    const int local = t - md.mom_begin;
    const int tr = local / md.mom_tiles_c, tc = local - (local / md.mom_tiles_c) * md.mom_tiles_c;
    const int r0 = tr * 64, c0 = tc * 64;
    const int m = g.m;
    float ss = 0.f;
    if (md.vec & 8) {
      // float32 rows, 16-byte aligned: each thread owns 4 consecutive columns of 4 rows
      const int tx4 = threadIdx.x & 15, ty = threadIdx.x >> 4;
      const int c = c0 + 4 * tx4;
      const float* Mp = reinterpret_cast<const float*>(md.m_ptr);
      const float* Gp = reinterpret_cast<const float*>(md.g_ptr);
      float4 mv[4], gv[4];
      bool ok[4];
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        const int r = r0 + ty + 16 * p;
        ok[p] = (r < md.rows) && (c < md.cols);
        mv[p] = make_float4(0.f, 0.f, 0.f, 0.f);
        gv[p] = mv[p];
        if (ok[p]) {
          mv[p] = *reinterpret_cast<const float4*>(Mp + (int64_t)r * md.m_ld + c);
          if (Gp) gv[p] = *reinterpret_cast<const float4*>(Gp + (int64_t)r * md.g_ld + c);
        }
      }
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        const int rr = ty + 16 * p, r = r0 + rr;
        float v[4] = {mv[p].x, mv[p].y, mv[p].z, mv[p].w};
        if (ok[p] && Gp) {
          const float gg[4] = {gv[p].x, gv[p].y, gv[p].z, gv[p].w};
#pragma unroll
          for (int k = 0; k < 4; ++k) v[k] = fmaf(beta, v[k], gg[k]);
          *reinterpret_cast<float4*>(reinterpret_cast<float*>(md.m_ptr) + (int64_t)r * md.m_ld + c) =
              make_float4(v[0], v[1], v[2], v[3]);
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) ss = fmaf(v[k], v[k], ss);
        if (!md.tall) {
          if (ok[p]) put_x0_4(g, bf, split, ((int64_t)md.z * m + r) * g.ldn + c, v);
        } else {
#pragma unroll
          for (int k = 0; k < 4; ++k) tile[rr][4 * tx4 + k] = v[k];
        }
      }
    } else {
      const int tx = threadIdx.x & 63, ty = threadIdx.x >> 6;
      for (int rr = ty; rr < 64; rr += 4) {
        const int r = r0 + rr, c = c0 + tx;
        float val = 0.f;
        if (r < md.rows && c < md.cols) {
          const int64_t idx = (int64_t)r * md.m_ld + c;
          float mv = load_as_f32(md.m_ptr, idx, md.m_dtype);
          if (md.g_ptr) {
            const float gv = load_as_f32(md.g_ptr, (int64_t)r * md.g_ld + c, md.g_dtype);
            mv = fmaf(beta, mv, gv);
            reinterpret_cast<float*>(md.m_ptr)[idx] = mv;
          }
          val = mv;
          if (!md.tall) put_x0(g, bf, split, ((int64_t)md.z * m + r) * g.ldn + c, val);
        }
        ss = fmaf(val, val, ss);
        if (md.tall) tile[rr][tx] = val;
      }
    }
    if (md.tall) {
      __syncthreads();
      // X0[c][r] = M[r][c]: the wide row index is the user column; lanes walk user rows
      const int tx = threadIdx.x & 63, ty = threadIdx.x >> 6;
      for (int cc = ty; cc < 64; cc += 4) {
        const int c = c0 + cc, r = r0 + tx;
        if (r < md.rows && c < md.cols) put_x0(g, bf, split, ((int64_t)md.z * m + c) * g.ldn + r, tile[tx][cc]);
      }
      __syncthreads();  // every warp has read the tile before any writes the next one
    }
    // the tile's sum of squares as one partial per warp (no block barrier), summed in a fixed order by
    // k_norm_finalize
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    if ((threadIdx.x & 31) == 0) partials[kMomSlots * t + (int)(threadIdx.x >> 5)] = ss;
  }
}

// s = 1 / (||M||_F + eps) (reading R4): one 256-thread CTA per matrix sums that matrix's per-warp tile
// partials, each thread a fixed strided share, then a fixed-order block reduction (deterministic).
__global__ void __launch_bounds__(256) k_norm_finalize(const Plan* plan, const int32_t* skip) {
  if (skip && *skip) return;
  const PlanHeader& h = plan->h;
  const int mi = blockIdx.x;
  if (mi >= h.n_mats) return;  // uniform over the CTA
  __shared__ float red[8];
  const MatDesc& md = h.mats[mi];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  float acc = 0.f;
  const float* part = h.partials + (int64_t)kMomSlots * md.mom_begin;
  const int n = kMomSlots * md.mom_count;
  for (int i = threadIdx.x; i < n; i += 256) acc += part[i];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) red[warp] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    float tot = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) tot += red[w];
    float sc = 1.f;
    if (!(h.flags & SMUON_NS_NO_NORMALIZE)) sc = 1.f / (sqrtf(tot) + h.eps);
    if (!isfinite(tot) && h.status) atomicOr(h.status, SMUON_DEV_NONFINITE_NORM);
    h.scale[mi] = sc;
  }
  if (warp == 0 && md.u_dtype == SMUON_BITS) {  // the message's pad words (past the last entry's word) are zero
    const int64_t nn = (int64_t)md.rows * md.cols;  // a multiple of 32
    const int64_t used = nn >> 5, total = ((nn + 127) >> 7) << 2;
    if (used + lane < total) reinterpret_cast<uint32_t*>(md.u_ptr)[used + lane] = 0u;
  }
}

// --------------------------------------------------------------------------
// Sign / pack / vote / update. Work unit: a chunk of 8 consecutive entries of
// one layer's row-major flattening; each layer's chunk range is padded to a
// multiple of 16 chunks (128 entries = 4 packed words), so the four lanes that
// build one packed word always belong to the same layer.
// --------------------------------------------------------------------------
__device__ __forceinline__ int find_layer(const EwTable* tb, int64_t chunk) {
  int lo = 0, hi = tb->n_layers - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (tb->layers[mid].chunk_begin <= chunk) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__device__ __forceinline__ int64_t ew_index(const EwLayer& L, int64_t e, int64_t ld) {
  // flat row-major entry -> element offset with a leading dimension
  if (ld == L.cols) return e;
  const int64_t r = e / L.cols;
  return r * ld + (e - r * L.cols);
}

// load 8 entries starting at flat entry e0 as float (missing entries -> +0)
__device__ __forceinline__ void load8(const void* p, int64_t ld, int32_t dtype, const EwLayer& L,
                                      int64_t e0, int vec, float* out) {
  if (vec && e0 + 8 <= L.n) {
    if (dtype == SMUON_BF16) {
      const uint4 w = *reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(p) + e0);
      const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        out[2 * k] = __uint_as_float(u[k] << 16);
        out[2 * k + 1] = __uint_as_float(u[k] & 0xffff0000u);
      }
    } else if (dtype == SMUON_F32) {
      const float4 a = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(p) + e0);
      const float4 b = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(p) + e0 + 4);
      out[0] = a.x; out[1] = a.y; out[2] = a.z; out[3] = a.w;
      out[4] = b.x; out[5] = b.y; out[6] = b.z; out[7] = b.w;
    } else {
      const uint2 w = *reinterpret_cast<const uint2*>(reinterpret_cast<const int8_t*>(p) + e0);
      const int8_t* q = reinterpret_cast<const int8_t*>(&w);
#pragma unroll
      for (int k = 0; k < 8; ++k) out[k] = (float)q[k];
    }
  } else {
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int64_t e = e0 + k;
      out[k] = (e < L.n) ? load_as_f32(p, ew_index(L, e, ld), dtype) : 0.f;
    }
  }
}

__device__ __forceinline__ void store8(void* p, int64_t ld, int32_t dtype, const EwLayer& L,
                                       int64_t e0, int vec, const float* v) {
  if (vec && e0 + 8 <= L.n) {
    if (dtype == SMUON_BF16) {
      uint4 w;
      w.x = pack_bf16x2_rn(v[0], v[1]); w.y = pack_bf16x2_rn(v[2], v[3]);
      w.z = pack_bf16x2_rn(v[4], v[5]); w.w = pack_bf16x2_rn(v[6], v[7]);
      *reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(p) + e0) = w;
    } else {
      float* q = reinterpret_cast<float*>(p) + e0;
      *reinterpret_cast<float4*>(q) = make_float4(v[0], v[1], v[2], v[3]);
      *reinterpret_cast<float4*>(q + 4) = make_float4(v[4], v[5], v[6], v[7]);
    }
  } else {
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int64_t e = e0 + k;
      if (e < L.n) store_from_f32(p, ew_index(L, e, ld), dtype, v[k]);
    }
  }
}

// combine the 8-bit sign bytes of lanes 4w..4w+3 into packed word w (reading R8)
__device__ __forceinline__ uint32_t gather_word(uint32_t byte, int lane) {
  uint32_t v = byte << (8 * (lane & 3));
  v |= __shfl_xor_sync(0xffffffffu, v, 1);
  v |= __shfl_xor_sync(0xffffffffu, v, 2);
  return v;
}

__device__ __forceinline__ int8_t threshold(int total, int tie) {
  return (int8_t)(total > 0 ? 1 : (total < 0 ? -1 : tie));
}

// sign bits (u >= 0: +0, -0 and positives; NaN is not) of 8 consecutive entries
__device__ __forceinline__ uint32_t pos_bits_bf16(const uint4 w) {
  const uint32_t u[4] = {w.x, w.y, w.z, w.w};
  uint32_t r = 0;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint32_t b = (u[k] >> (16 * h)) & 0xffffu;
      const uint32_t mag = b & 0x7fffu;
      const bool pos = (mag == 0u) || (!(b & 0x8000u) && mag <= 0x7f80u);
      r |= (uint32_t)pos << (2 * k + h);
    }
  }
  return r;
}

__device__ __forceinline__ uint32_t pos_bits_f32(const float* u) {
  uint32_t r = 0;
#pragma unroll
  for (int k = 0; k < 8; ++k) r |= (uint32_t)(u[k] >= 0.f) << k;
  return r;
}

// the 8 sign bits of one worker's entries e0..e0+7 (entries past the end -> 0)
template <bool kBf16>
__device__ __forceinline__ uint32_t worker_bits(const EwSrc& S, const EwLayer& L, int64_t e0, int32_t dtype) {
  if (L.vec && e0 + 8 <= L.n) {
    if (kBf16) return pos_bits_bf16(*reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(S.ptr) + e0));
    const float4 a = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(S.ptr) + e0);
    const float4 b = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(S.ptr) + e0 + 4);
    const float u[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    return pos_bits_f32(u);
  }
  uint32_t r = 0;
  for (int k = 0; k < 8; ++k) {
    const int64_t e = e0 + k;
    if (e < L.n) r |= (uint32_t)(load_as_f32(S.ptr, ew_index(L, e, S.ld), dtype) >= 0.f) << k;
  }
  return r;
}

// layer of each lane's chunk: one binary search per warp, then a short forward walk
__device__ __forceinline__ int warp_layer(const EwTable& tb, int64_t wbase, int64_t chunk, int lane) {
  int l0 = 0;
  if (lane == 0) l0 = find_layer(&tb, wbase);
  l0 = __shfl_sync(0xffffffffu, l0, 0);
  int l = l0;
  while (l + 1 < tb.n_layers && tb.layers[l + 1].chunk_begin <= chunk) ++l;
  return l;
}

// SignMuon summary, flow steps 2-4 fused: sign (U >= 0), optional packed
// message, majority vote (sum = 2*popcount - M over per-entry worker masks, or
// the integer sum of +-1), then W <- W - eta*vote in float32, rounded to W's
// type. Work unit: 8 consecutive entries per lane.
// per 16-bit lane of w: 1 where the bf16 value is >= 0 (+0, -0, positives; not NaN)
// Plain integer arithmetic on both halves at once (no carries cross the halves):
// with mag = h & 0x7fff, u >= 0 holds iff (sign clear and mag <= 0x7f80, i.e.
// not a NaN) or mag == 0 (-0). Bit 15 of mag + 0x7f is clear iff mag <= 0x7f80;
// bit 15 of mag + 0x7fff is clear iff mag == 0.
__device__ __forceinline__ uint32_t pos_halves_bf16(uint32_t w) {
  const uint32_t mag = w & 0x7fff7fffu;
  const uint32_t le = mag + 0x007f007fu;
  const uint32_t nz = mag + 0x7fff7fffu;
  return (((~le & ~w) | ~nz) >> 15) & 0x00010001u;
}

// 256-bit accesses for a lane's 16 bf16 entries (32 bytes, whole sectors) where the address allows
__device__ __forceinline__ void ld_v8_b32(const void* p, uint32_t* u) {
  asm volatile("ld.global.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]), "=r"(u[7])
               : "l"(p));
}
__device__ __forceinline__ void st_v8_b32(void* p, const uint32_t* u) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};"
               ::"l"(p), "r"(u[0]), "r"(u[1]), "r"(u[2]), "r"(u[3]), "r"(u[4]), "r"(u[5]), "r"(u[6]), "r"(u[7])
               : "memory");
}

// vote and update of 8 entries e0..e0+7 from their 4 packed count words, W
// already loaded into w (when kHasW); kStoreW false leaves the updated w to the caller's store
template <bool kHasW, bool kStoreW = true>
__device__ __forceinline__ void vote_apply8(const EwTable& tb, const EwLayer& L, int64_t e0, const uint32_t* cnt,
                                            float* w) {
  int8_t v8[8];
  // eta * v for v = +1, -1 and the tie value: exact products, chosen per entry
  const float up = tb.eta, down = -tb.eta, tied = tb.eta * (float)tb.tie;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const int c2 = 2 * (int)((cnt[k >> 1] >> (16 * (k & 1))) & 0xffffu);
    v8[k] = (int8_t)(c2 > tb.M ? 1 : (c2 < tb.M ? -1 : tb.tie));
    w[k] = __fsub_rn(w[k], c2 > tb.M ? up : (c2 < tb.M ? down : tied));
  }
  if (kHasW && kStoreW) store8(L.w, L.w_ld, L.w_dtype, L, e0, 1, w);  // no W: signs, message and vote only
  if (L.vote_out) {
    int8_t* dst = L.vote_out + e0;
    if ((reinterpret_cast<uintptr_t>(dst) & 7) == 0) {
      uint2 pk;
      memcpy(&pk, v8, 8);
      *reinterpret_cast<uint2*>(dst) = pk;
    } else {
#pragma unroll
      for (int k = 0; k < 8; ++k) dst[k] = v8[k];
    }
  }
}

template <bool kHasW>
__device__ __forceinline__ void vote_finish8(const EwTable& tb, const EwLayer& L, int64_t e0, const uint32_t* cnt) {
  // W is loaded only here, after the workers' loads: fewer live registers, so
  // three CTAs fit per SM (more loads in flight hide more latency)
  float w[8];
  if (kHasW) load8(L.w, L.w_ld, L.w_dtype, L, e0, 1, w);
  vote_apply8<kHasW>(tb, L, e0, cnt, w);
}

// int8 (integer-sum) vote on bf16 outputs: the count of positive signs of each
// entry is accumulated two entries per 32-bit add (16-bit lanes), then
// sum = 2 * count - M (the +-1 sum of the all-reduce variant). Each lane takes
// two consecutive 8-entry chunks (16 entries, 16-byte loads per worker); layer
// chunk ranges are multiples of 16 chunks, so a pair never straddles layers.
template <bool kHasW>
__device__ __forceinline__ void vote_update_int8_bf16(const EwTable& tb) {
  const int lane = threadIdx.x & 31;
  const int64_t warp_global = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t warps_total = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const int M = tb.M;
  for (int64_t wbase = warp_global * 64; wbase < tb.total_chunks; wbase += warps_total * 64) {
    const int64_t chunk = wbase + 2 * lane;
    const bool active = chunk < tb.total_chunks;
    const int li = warp_layer(tb, wbase, active ? chunk : tb.total_chunks - 1, lane);
    const EwLayer& L = tb.layers[li];
    const int64_t e0 = (chunk - L.chunk_begin) * 8;
    if (!(active && e0 < L.n)) continue;
    if (L.vec && e0 + 16 <= L.n) {
      uint32_t cnt[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
      for (int wk0 = 0; wk0 < M; wk0 += 4) {
        uint4 u[4][2];
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (wk0 + j < M) {
            const uint4* p = reinterpret_cast<const uint4*>(
                reinterpret_cast<const __nv_bfloat16*>(tb.srcs[L.src_first + wk0 + j].ptr) + e0);
            u[j][0] = p[0];
            u[j][1] = p[1];
          }
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (wk0 + j < M) {
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              cnt[4 * hh + 0] += pos_halves_bf16(u[j][hh].x);
              cnt[4 * hh + 1] += pos_halves_bf16(u[j][hh].y);
              cnt[4 * hh + 2] += pos_halves_bf16(u[j][hh].z);
              cnt[4 * hh + 3] += pos_halves_bf16(u[j][hh].w);
            }
          }
      }
      vote_finish8<kHasW>(tb, L, e0, cnt);
      vote_finish8<kHasW>(tb, L, e0 + 8, cnt + 4);
    } else {
      // ragged or strided layers: entry by entry
      const int nent = (int)min((int64_t)16, L.n - e0);
      for (int k = 0; k < nent; ++k) {
        const int64_t e = e0 + k;
        int c = 0;
        for (int wk = 0; wk < M; ++wk) {
          const EwSrc& S = tb.srcs[L.src_first + wk];
          c += load_as_f32(S.ptr, ew_index(L, e, S.ld), SMUON_BF16) >= 0.f ? 1 : 0;
        }
        const int8_t v = threshold(2 * c - M, tb.tie);
        if (L.w) {
          const int64_t wi = ew_index(L, e, L.w_ld);
          store_from_f32(L.w, wi, L.w_dtype, __fsub_rn(load_as_f32(L.w, wi, L.w_dtype), tb.eta * (float)v));
        }
        if (L.vote_out) L.vote_out[e] = v;
      }
    }
  }
}

// int8 sum-then-sign vote on int8 sign matrices (the signs written by a
// Newton-Schulz call with an I8 output): an entry counts as positive when its
// sign bit is clear (+1, and 0 by the u >= 0 rule). Each lane takes 16
// consecutive entries, one 16-byte load per worker; the positive flags add
// up per byte (M <= 64, no carries), and the byte counts are spread into the
// 16-bit lanes vote_finish8 takes.
template <bool kHasW>
__device__ __forceinline__ void vote_update_i8src(const EwTable& tb) {
  const int lane = threadIdx.x & 31;
  const int64_t warp_global = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t warps_total = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const int M = tb.M;
  for (int64_t wbase = warp_global * 64; wbase < tb.total_chunks; wbase += warps_total * 64) {
    const int64_t chunk = wbase + 2 * lane;
    const bool active = chunk < tb.total_chunks;
    const int li = warp_layer(tb, wbase, active ? chunk : tb.total_chunks - 1, lane);
    const EwLayer& L = tb.layers[li];
    const int64_t e0 = (chunk - L.chunk_begin) * 8;
    if (!(active && e0 < L.n)) continue;
    if (L.vec && e0 + 16 <= L.n) {
      // W first: the int8 signs need few registers, so W's loads go out together with the workers'
      float w[16];
      __nv_bfloat16* wb = reinterpret_cast<__nv_bfloat16*>(L.w) + e0;
      const bool w32 = kHasW && L.w_dtype == SMUON_BF16 && (reinterpret_cast<uintptr_t>(wb) & 31) == 0;
      if (w32) {  // the lane's 16 bf16 as one 32-byte sector
        uint32_t u[8];
        ld_v8_b32(wb, u);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          w[2 * k] = __uint_as_float(u[k] << 16);
          w[2 * k + 1] = __uint_as_float(u[k] & 0xffff0000u);
        }
      } else if (kHasW) {
        load8(L.w, L.w_ld, L.w_dtype, L, e0, 1, w);
        load8(L.w, L.w_ld, L.w_dtype, L, e0 + 8, 1, w + 8);
      }
      uint32_t b[4] = {0u, 0u, 0u, 0u};  // per byte: positive signs of entries e0 + 4i .. e0 + 4i + 3
      for (int wk0 = 0; wk0 < M; wk0 += 4) {  // four workers' 16-byte loads in flight (16 registers)
        uint4 u[4];
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (wk0 + j < M) u[j] = *reinterpret_cast<const uint4*>(
                               reinterpret_cast<const int8_t*>(tb.srcs[L.src_first + wk0 + j].ptr) + e0);
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (wk0 + j < M) {
            b[0] += (~u[j].x >> 7) & 0x01010101u;
            b[1] += (~u[j].y >> 7) & 0x01010101u;
            b[2] += (~u[j].z >> 7) & 0x01010101u;
            b[3] += (~u[j].w >> 7) & 0x01010101u;
          }
      }
      uint32_t cnt[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        cnt[2 * i] = __byte_perm(b[i], 0u, 0x4140);      // entries 4i, 4i + 1 in the low and high halves
        cnt[2 * i + 1] = __byte_perm(b[i], 0u, 0x4342);  // entries 4i + 2, 4i + 3
      }
      if (w32) {
        vote_apply8<kHasW, false>(tb, L, e0, cnt, w);
        vote_apply8<kHasW, false>(tb, L, e0 + 8, cnt + 4, w + 8);
        uint32_t u[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) u[k] = pack_bf16x2_rn(w[2 * k], w[2 * k + 1]);
        st_v8_b32(wb, u);
      } else {
        vote_apply8<kHasW>(tb, L, e0, cnt, w);
        vote_apply8<kHasW>(tb, L, e0 + 8, cnt + 4, w + 8);
      }
    } else {
      const int nent = (int)min((int64_t)16, L.n - e0);
      for (int k = 0; k < nent; ++k) {
        const int64_t e = e0 + k;
        int c = 0;
        for (int wk = 0; wk < M; ++wk) {
          const EwSrc& S = tb.srcs[L.src_first + wk];
          c += reinterpret_cast<const int8_t*>(S.ptr)[ew_index(L, e, S.ld)] >= 0 ? 1 : 0;
        }
        const int8_t v = threshold(2 * c - M, tb.tie);
        if (L.w) {
          const int64_t wi = ew_index(L, e, L.w_ld);
          store_from_f32(L.w, wi, L.w_dtype, __fsub_rn(load_as_f32(L.w, wi, L.w_dtype), tb.eta * (float)v));
        }
        if (L.vote_out) L.vote_out[e] = v;
      }
    }
  }
}

// the 16 message bits of one lane (bit j = entry e0 + j is >= 0) from the
// per-half flags of its 8 words (bit 0: entry 2i, bit 16: entry 2i + 1)
__device__ __forceinline__ uint32_t mask16_from_halves(const uint32_t* p) {
  uint32_t y = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) y |= p[i] << (2 * i);
  return (y | (y >> 15)) & 0xffffu;
}

// per-half sign flags of entries e, e + 1 (only those below `left` entries), one by one
__device__ __noinline__ uint32_t pos_halves_scalar(const EwSrc& S, const EwLayer& L, int64_t e, int left) {
  uint32_t f = 0;
  if (left > 0) f |= (uint32_t)(load_as_f32(S.ptr, ew_index(L, e, S.ld), SMUON_BF16) >= 0.f);
  if (left > 1) f |= (uint32_t)(load_as_f32(S.ptr, ew_index(L, e + 1, S.ld), SMUON_BF16) >= 0.f) << 16;
  return f;
}

// vote and update of entries e, e + 1 (only those below `left`) from their packed counts
__device__ __noinline__ void finish_pair_scalar(const EwTable& tb, const EwLayer& L, int64_t e, int left,
                                                uint32_t cnt) {
  for (int k = 0; k < 2 && k < left; ++k) {
    const int c = (int)((cnt >> (16 * k)) & 0xffffu);
    const int8_t v = threshold(2 * c - tb.M, tb.tie);
    if (L.w) {
      const int64_t wi = ew_index(L, e + k, L.w_ld);
      store_from_f32(L.w, wi, L.w_dtype, __fsub_rn(load_as_f32(L.w, wi, L.w_dtype), tb.eta * (float)v));
    }
    if (L.vote_out) L.vote_out[e + k] = v;
  }
}

// Fused sign / 1-bit message / majority vote / update for bf16 outputs, any
// M up to 64, 16 entries per lane. Per worker, the lane's 16 sign flags (U >= 0)
// are kept as 8 words of per-half flags. Their sum over the workers is, per
// entry, the number of set bits among the M workers' message bits (two 16-bit
// counters per add): the popcount of the entry's bits, and sum = 2*count - M.
// The same flags are the lane's 16 message bits; two neighbouring lanes join
// theirs into one packed word (entry i -> bit i%32 of word i/32) with one
// shuffle. Layer chunk ranges are multiples of 16 chunks (128 entries), so a
// lane pair never straddles a layer and the even lane's e0 is a multiple of 32.
template <bool kHasW>
__device__ __forceinline__ void vote_update_bf16x16(const EwTable& tb) {
  const int lane = threadIdx.x & 31;
  const int64_t warp_global = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t warps_total = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const int M = tb.M;
  const bool any_packed = tb.any_packed != 0;  // uniform: the shuffles below involve every lane
  for (int64_t wbase = warp_global * 64; wbase < tb.total_chunks; wbase += warps_total * 64) {
    const int64_t chunk = wbase + 2 * lane;
    const bool active = chunk < tb.total_chunks;
    const int li = warp_layer(tb, wbase, active ? chunk : tb.total_chunks - 1, lane);
    const EwLayer& L = tb.layers[li];
    const int64_t e0 = (chunk - L.chunk_begin) * 8;
    const bool live = active && e0 < L.n;
    const bool fast = live && L.vec && e0 + 16 <= L.n;
    const int nent = live ? (int)min((int64_t)16, L.n - e0) : 0;
    uint32_t cnt[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
    for (int wk0 = 0; wk0 < M; wk0 += 4) {
      uint4 u[4][2];
      if (fast) {
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (wk0 + j < M) {
            const uint4* q = reinterpret_cast<const uint4*>(
                reinterpret_cast<const __nv_bfloat16*>(tb.srcs[L.src_first + wk0 + j].ptr) + e0);
            u[j][0] = q[0];
            u[j][1] = q[1];
          }
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int wk = wk0 + j;
        if (wk >= M) break;  // uniform across the warp
        uint32_t f[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
        if (fast) {
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            f[4 * hh + 0] = pos_halves_bf16(u[j][hh].x);
            f[4 * hh + 1] = pos_halves_bf16(u[j][hh].y);
            f[4 * hh + 2] = pos_halves_bf16(u[j][hh].z);
            f[4 * hh + 3] = pos_halves_bf16(u[j][hh].w);
          }
        } else if (live) {  // ragged tail or strided layer: entry by entry
          const EwSrc& S = tb.srcs[L.src_first + wk];
#pragma unroll
          for (int i = 0; i < 8; ++i) f[i] = pos_halves_scalar(S, L, e0 + 2 * i, nent - 2 * i);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) cnt[i] += f[i];
        if (any_packed) {
          uint32_t v = mask16_from_halves(f) << (16 * (lane & 1));
          v |= __shfl_xor_sync(0xffffffffu, v, 1);
          if (active && L.packed_out && (lane & 1) == 0) L.packed_out[(int64_t)wk * L.words + (e0 >> 5)] = v;
        }
      }
    }
    if (!live) continue;
    if (fast) {
      vote_finish8<kHasW>(tb, L, e0, cnt);
      vote_finish8<kHasW>(tb, L, e0 + 8, cnt + 4);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) finish_pair_scalar(tb, L, e0 + 2 * i, nent - 2 * i, cnt[i]);
    }
  }
}

template <bool kPopcount, bool kBf16, typename MaskT>
__device__ __forceinline__ void vote_update_body(const EwTable& tb) {
  const int lane = threadIdx.x & 31;
  const int64_t warp_global = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t warps_total = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const int M = tb.M;
  for (int64_t wbase = warp_global * 32; wbase < tb.total_chunks; wbase += warps_total * 32) {
    const int64_t chunk = wbase + lane;
    const bool active = chunk < tb.total_chunks;
    const int li = warp_layer(tb, wbase, active ? chunk : tb.total_chunks - 1, lane);
    const EwLayer& L = tb.layers[li];
    const int64_t e0 = (chunk - L.chunk_begin) * 8;
    const bool live = active && e0 < L.n;
    float w[8];
    if (live && L.w) load8(L.w, L.w_ld, L.w_dtype, L, e0, L.vec, w);
    MaskT mask[8];
    int sum[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) { mask[k] = 0; sum[k] = 0; }
    for (int wk0 = 0; wk0 < M; wk0 += 4) {
      uint32_t bits[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int wk = wk0 + j;
        bits[j] = (wk < M && live) ? worker_bits<kBf16>(tb.srcs[L.src_first + wk], L, e0, tb.src_dtype) : 0u;
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int wk = wk0 + j;
        if (wk >= M) break;  // uniform across the warp
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint32_t pos = (bits[j] >> k) & 1u;
          if (kPopcount) mask[k] |= (MaskT)pos << wk;
          else sum[k] += pos ? 1 : -1;
        }
        if (tb.any_packed) {  // warp-uniform: every lane takes part in the shuffles
          const uint32_t word = gather_word(bits[j], lane);
          if (active && L.packed_out && (lane & 3) == 0)
            L.packed_out[(int64_t)wk * L.words + ((chunk - L.chunk_begin) >> 2)] = word;
        }
      }
    }
    if (!live) continue;
    int8_t v8[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int cnt = sizeof(MaskT) == 8 ? __popcll((unsigned long long)mask[k]) : __popc((unsigned)mask[k]);
      const int total = kPopcount ? 2 * cnt - M : sum[k];
      v8[k] = threshold(total, tb.tie);
      w[k] = __fsub_rn(w[k], tb.eta * (float)v8[k]);
    }
    if (L.w) store8(L.w, L.w_ld, L.w_dtype, L, e0, L.vec, w);
    if (L.vote_out) {
      if (e0 + 8 <= L.n && ((reinterpret_cast<uintptr_t>(L.vote_out + e0) & 7) == 0)) {
        uint2 pk;
        memcpy(&pk, v8, 8);
        *reinterpret_cast<uint2*>(L.vote_out + e0) = pk;
      } else {
        for (int k = 0; k < 8; ++k) if (e0 + k < L.n) L.vote_out[e0 + k] = v8[k];
      }
    }
  }
}

// Vote and update from the workers' 1-bit messages (SignMuon summary, flow steps 3-4, all-gather
// variant): the message words of a Newton-Schulz call with a BITS output or of an all-gather. One
// lane per packed word, i.e. 32 consecutive entries: the M words (M/8 bytes per entry) are added
// bit-sliced -- plane p holds bit p of every entry's count of set bits, as many planes as M needs --
// by a ripple of half adders per worker, and the counts are compared with h = floor(M/2) plane by
// plane from the top:
// count > h is the +1 vote (2*count > M), count == h with M even the tie, the rest -1. Bits past a
// layer's last entry are zero and are never applied. Layer chunk ranges are multiples of 16 chunks
// (4 words), so global word g is chunk 4g.
template <bool kHasW, int kPlanes>
__device__ __forceinline__ void vote_update_bits(const EwTable& tb) {
  const int lane = threadIdx.x & 31;
  const int64_t warp_global = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t warps_total = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const int M = tb.M;
  const int h = M >> 1;
  const uint32_t even = (M & 1) ? 0u : 0xffffffffu;
  const int64_t total_words = tb.total_chunks >> 2;
  for (int64_t wbase = warp_global * 32; wbase < total_words; wbase += warps_total * 32) {
    const int64_t gw = wbase + lane;
    const bool active = gw < total_words;
    const int li = warp_layer(tb, 4 * wbase, active ? 4 * gw : tb.total_chunks - 1, lane);
    const EwLayer& L = tb.layers[li];
    const int64_t w = gw - (L.chunk_begin >> 2);
    const int64_t e0 = 32 * w;
    const bool lane_ok = active && e0 < L.n;
    const int nent = lane_ok ? (int)min((int64_t)32, L.n - e0) : 0;
    const bool fast = L.vec && nent == 32;
    // the warp's 32 words (1024 entries) whole and in one contiguous layer: W then moves in coalesced
    // 512-byte rows (lane l holds entries 8 (32 q + l) .. + 7 of load q), requested before the message
    // words, and each lane takes its vote bits from the lane that counted them
    // (every lane executes both warp intrinsics: neither sits behind a lane-dependent condition)
    const int li0 = __shfl_sync(0xffffffffu, li, 0);
    const bool warp_fast = __all_sync(0xffffffffu, fast && li == li0);
    const bool pre_w = kHasW && warp_fast && L.w_dtype == SMUON_BF16;  // warp-uniform
    const int64_t ebase = e0 - 32 * lane;                                 // the warp's first entry
    uint4 wq[4];
    if (pre_w) {
      const uint4* wp = reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(L.w) + ebase);
#pragma unroll
      for (int q = 0; q < 4; ++q) wq[q] = wp[32 * q + lane];
    }
    if (!lane_ok) continue;  // never taken on the warp-wide path (every lane is whole there)
    uint32_t c[kPlanes];  // counts up to M need kPlanes planes (4 for M <= 15, 7 for M <= 64)
#pragma unroll
    for (int p = 0; p < kPlanes; ++p) c[p] = 0u;
    for (int wk0 = 0; wk0 < M; wk0 += 8) {
      uint32_t x[8];
#pragma unroll
      for (int j = 0; j < 8; ++j)
        x[j] = (wk0 + j < M) ? reinterpret_cast<const uint32_t*>(tb.srcs[L.src_first + wk0 + j].ptr)[w] : 0u;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        uint32_t carry = x[j];
#pragma unroll
        for (int p = 0; p < kPlanes; ++p) {
          const uint32_t t = c[p] & carry;
          c[p] ^= carry;
          carry = t;
        }
      }
    }
    uint32_t gt = 0u, eq = 0xffffffffu;
#pragma unroll
    for (int p = kPlanes - 1; p >= 0; --p) {
      if ((h >> p) & 1) {
        eq &= c[p];
      } else {
        gt |= eq & c[p];
        eq &= ~c[p];
      }
    }
    const uint32_t pos = gt, tie = eq & even;
    const float up = tb.eta, down = -tb.eta, tied = tb.eta * (float)tb.tie;
    if (pre_w) {
      __nv_bfloat16* wout = reinterpret_cast<__nv_bfloat16*>(L.w) + ebase;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        // entries 8 (32 q + lane) .. + 7: byte (lane & 3) of the word counted by lane 8 q + lane / 4
        const int src = 8 * q + (lane >> 2), sh = 8 * (lane & 3);
        const uint32_t pb = __shfl_sync(0xffffffffu, pos, src) >> sh;
        const uint32_t tbits = __shfl_sync(0xffffffffu, tie, src) >> sh;
        const uint32_t u[4] = {wq[q].x, wq[q].y, wq[q].z, wq[q].w};
        float wv[8];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          wv[2 * k] = __uint_as_float(u[k] << 16);
          wv[2 * k + 1] = __uint_as_float(u[k] & 0xffff0000u);
        }
#pragma unroll
        for (int k = 0; k < 8; ++k)
          wv[k] = __fsub_rn(wv[k], ((pb >> k) & 1u) ? up : (((tbits >> k) & 1u) ? tied : down));
        uint4 o;
        o.x = pack_bf16x2_rn(wv[0], wv[1]); o.y = pack_bf16x2_rn(wv[2], wv[3]);
        o.z = pack_bf16x2_rn(wv[4], wv[5]); o.w = pack_bf16x2_rn(wv[6], wv[7]);
        reinterpret_cast<uint4*>(wout)[32 * q + lane] = o;
      }
      if (L.vote_out) {  // this lane's own 32 entries
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          const uint32_t pb = pos >> (8 * g), tbits = tie >> (8 * g);
          int8_t v8[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) v8[k] = (int8_t)(((pb >> k) & 1u) ? 1 : (((tbits >> k) & 1u) ? tb.tie : -1));
          int8_t* dst = L.vote_out + e0 + 8 * g;
          if ((reinterpret_cast<uintptr_t>(dst) & 7) == 0) {
            uint2 pk;
            memcpy(&pk, v8, 8);
            *reinterpret_cast<uint2*>(dst) = pk;
          } else {
#pragma unroll
            for (int k = 0; k < 8; ++k) dst[k] = v8[k];
          }
        }
      }
    } else if (fast) {
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        float wv[8];
        int8_t v8[8];
        if (kHasW) load8(L.w, L.w_ld, L.w_dtype, L, e0 + 8 * g, 1, wv);
        const uint32_t pb = pos >> (8 * g), tbits = tie >> (8 * g);
        if (kHasW) {
#pragma unroll
          for (int k = 0; k < 8; ++k)
            wv[k] = __fsub_rn(wv[k], ((pb >> k) & 1u) ? up : (((tbits >> k) & 1u) ? tied : down));
          store8(L.w, L.w_ld, L.w_dtype, L, e0 + 8 * g, 1, wv);
        }
        if (L.vote_out) {
#pragma unroll
          for (int k = 0; k < 8; ++k) v8[k] = (int8_t)(((pb >> k) & 1u) ? 1 : (((tbits >> k) & 1u) ? tb.tie : -1));
          int8_t* dst = L.vote_out + e0 + 8 * g;
          if ((reinterpret_cast<uintptr_t>(dst) & 7) == 0) {
            uint2 pk;
            memcpy(&pk, v8, 8);
            *reinterpret_cast<uint2*>(dst) = pk;
          } else {
#pragma unroll
            for (int k = 0; k < 8; ++k) dst[k] = v8[k];
          }
        }
      }
    } else {  // ragged last word or strided W: entry by entry
      for (int j = 0; j < nent; ++j) {
        const int64_t e = e0 + j;
        const bool p1 = (pos >> j) & 1u, t1 = (tie >> j) & 1u;
        const int8_t v = (int8_t)(p1 ? 1 : (t1 ? tb.tie : -1));
        if (kHasW) {
          const int64_t wi = ew_index(L, e, L.w_ld);
          store_from_f32(L.w, wi, L.w_dtype, __fsub_rn(load_as_f32(L.w, wi, L.w_dtype), tb.eta * (float)v));
        }
        if (L.vote_out) L.vote_out[e] = v;
      }
    }
  }
}

template <bool kHasW, int kPlanes>
__global__ void __launch_bounds__(256, 4) k_vote_update_bits(const __grid_constant__ EwTable tb) {
  vote_update_bits<kHasW, kPlanes>(tb);
}

// ---- 1-bit vote and update with the operands staged by the bulk-copy engine
// The same vote as vote_update_bits, for bf16 W: one elected lane streams each block's W rows (8192 entries,
// 16 KB) and its M message rows (256 words each) into a ring of shared-memory slots with cp.async.bulk,
// so the copies of the next slots are in flight while eight consumer warps count, vote and write W back
// from the current one. Every wait is bounded: when one runs out the CTA records SMUON_DEV_WAIT_TIMEOUT in
// the caller's d_status, stops, waits (bounded) for the copies it issued and returns.
namespace bitsq {
constexpr int kWords = 256;               // packed words per block (one per consumer lane)
constexpr int kEntries = 32 * kWords;     // 8192
constexpr int kWBytes = 2 * kEntries;     // bf16 W of one block
constexpr int kSlots = 3;
constexpr int kConsumers = 8;             // warps
constexpr int kThreads = 32 * (kConsumers + 1);
constexpr int kMaxM = 16;
constexpr unsigned long long kBudget = 1ull << 32;  // about 2 s of SM clock
constexpr unsigned long long kTestBudget = 1ull << 16;
__host__ __device__ constexpr int slot_bytes(int M) { return kWBytes + M * kWords * 4; }
// the subtrahends of four entries for each (+1 bits, zero bits) pair, in eight copies: copy r serves the
// lanes with lane % 8 == r, and entry i of copy r sits in 16-byte unit 8 i + r, so the eight lanes of a
// quarter warp (one shared-memory wavefront of 16-byte loads) always read eight different bank groups
constexpr int kLutBytes = 8 * 256 * 16;
__host__ __device__ constexpr int smem_bytes(int M) {
  return kSlots * slot_bytes(M) + kLutBytes + 16 * kSlots + 8 * (kEwMaxLayers + 1) + 16;
}

__device__ __forceinline__ uint32_t saddr(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }
__device__ __forceinline__ void bar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}
__device__ __forceinline__ void bar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void bar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool bar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
  return ok != 0;
}
// bounded wait: false when the budget ran out or another role gave up
__device__ __forceinline__ bool bar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                         unsigned long long budget) {
  if (bar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = clock64();
  for (uint32_t i = 1;; ++i) {
    if (bar_try_wait(bar, parity)) return true;
    if ((i & 63) == 0 && (*abort_flag || clock64() - t0 > budget)) return false;
  }
}
// full adder over bit planes: s = a ^ b ^ c, carry = majority(a, b, c) (one three-input logic op each)
__device__ __forceinline__ void full_add(uint32_t a, uint32_t b, uint32_t c, uint32_t& s, uint32_t& carry) {
  s = a ^ b ^ c;
  carry = (a & b) | (c & (a ^ b));
}
// per bit position, the number of set bits among x[0..7] as planes q[0] (1) .. q[3] (8)
__device__ __forceinline__ void csa_count8(const uint32_t (&x)[8], uint32_t (&q)[4]) {
  uint32_t sa, ca, sb, cb, sc, cc, se, ce;
  full_add(x[0], x[1], x[2], sa, ca);   // weight 1 -> 1, 2
  full_add(x[3], x[4], x[5], sb, cb);
  full_add(sa, sb, x[6], sc, cc);
  q[0] = sc ^ x[7];
  const uint32_t cd = sc & x[7];
  full_add(ca, cb, cc, se, ce);         // weight 2 -> 2, 4
  q[1] = se ^ cd;
  const uint32_t cf = se & cd;
  q[2] = ce ^ cf;                       // weight 4 -> 4, 8
  q[3] = ce & cf;
}
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               ::"r"(dst), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar) : "memory");
}
}  // namespace bitsq

template <int kPlanes>
__global__ void __launch_bounds__(bitsq::kThreads) k_vote_update_bits_tma(const __grid_constant__ EwTable tb) {
  using namespace bitsq;
  extern __shared__ __align__(128) unsigned char sm[];
  const int M = tb.M;
  const int SB = slot_bytes(M);
  unsigned char* ring = sm;
  float4* lut = reinterpret_cast<float4*>(sm + kSlots * SB);
  const uint32_t bars = saddr(sm + kSlots * SB + kLutBytes);  // full[kSlots], empty[kSlots]
  int64_t* blk = reinterpret_cast<int64_t*>(sm + kSlots * SB + kLutBytes + 16 * kSlots);  // block prefix per layer
  volatile int* abort_flag = reinterpret_cast<volatile int*>(blk + kEwMaxLayers + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int q = 0; q < kSlots; ++q) {
      bar_init(bars + 8 * q, 1);
      bar_init(bars + 8 * (kSlots + q), kConsumers);
    }
    int64_t acc = 0;
    for (int l = 0; l < tb.n_layers; ++l) {
      blk[l] = acc;
      acc += (tb.layers[l].words + kWords - 1) / kWords;
    }
    blk[tb.n_layers] = acc;
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  // lut[p | z << 4]: entry e of four (bit e of p: a +1 vote after the tie rule, bit e of z: a zero vote)
  // subtracts eta, 0 or -eta
  for (int t = threadIdx.x; t < 8 * 256; t += blockDim.x) {
    const int i = t >> 3;
    float d[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) d[e] = ((i >> (4 + e)) & 1) ? 0.f : (((i >> e) & 1) ? tb.eta : -tb.eta);
    lut[t] = make_float4(d[0], d[1], d[2], d[3]);
  }
  __syncthreads();
  const int64_t total = blk[tb.n_layers];
  const unsigned long long budget = tb.test_starve ? kTestBudget : kBudget;
  // block g: its layer (every role walks the blocks in increasing order, so the layer only moves forward)
  // and the block's index within that layer
  auto locate = [&](int64_t g, int& li, int64_t& b) {
    while (li + 1 < tb.n_layers && blk[li + 1] <= g) ++li;
    b = g - blk[li];
  };
  bool ok = true;
  if (warp == kConsumers) {
    // ---------------- producer (one lane)
    if (lane == 0) {
      int s = 0, li = 0;
      uint32_t ph = 0, armed = 0, last_par = 0;
      for (int64_t g = blockIdx.x; g < total && !tb.test_starve; g += gridDim.x) {
        if (!bar_wait(bars + 8 * (kSlots + s), ph ^ 1u, abort_flag, budget)) { ok = false; break; }
        int64_t b;
        locate(g, li, b);
        const EwLayer& L = tb.layers[li];
        const int ne = (int)min((int64_t)kEntries, L.n - b * kEntries);      // a multiple of 8
        const int nw = (int)min((int64_t)kWords, L.words - b * kWords);      // a multiple of 4
        const uint32_t full = bars + 8 * s;
        bar_expect_tx(full, (uint32_t)(2 * ne + M * 4 * nw));
        armed |= 1u << s;
        last_par = (last_par & ~(1u << s)) | (ph << s);
        const uint32_t dst = saddr(ring + (size_t)s * SB);
        bulk_load(dst, reinterpret_cast<const __nv_bfloat16*>(L.w) + b * kEntries, (uint32_t)(2 * ne), full);
        for (int k = 0; k < M; ++k)
          bulk_load(dst + kWBytes + k * kWords * 4,
                    reinterpret_cast<const uint32_t*>(tb.srcs[L.src_first + k].ptr) + b * kWords,
                    (uint32_t)(4 * nw), full);
        if (++s == kSlots) { s = 0; ph ^= 1u; }
      }
      if (!ok) {
        *abort_flag = 1;
        if (tb.status) atomicOr(tb.status, SMUON_DEV_WAIT_TIMEOUT);
      }
      // the copies this lane issued land before the CTA leaves
      for (int q = 0; q < kSlots; ++q)
        if (armed & (1u << q)) {
          const unsigned long long t0 = clock64();
          while (!bar_try_wait(bars + 8 * q, (last_par >> q) & 1u) && clock64() - t0 < kBudget) {}
        }
    }
  } else {
    // ---------------- consumers: lane = one packed word of the block (32 entries)
    const int h = M >> 1;
    const uint32_t even = (M & 1) ? 0u : 0xffffffffu;
    // the tie rule folded into two masks per word: ties vote +1 with tie_value 1 (they join the +1 mask), -1
    // with tie_value -1 (they stay out of it) and 0 with tie_value 0 (W unchanged: the zero mask, which only
    // an even M can produce; a grid-uniform switch)
    const bool zero_ties = tb.tie == 0 && !(M & 1);
    const int j = warp * 32 + lane;
    int s = 0, li = 0;
    uint32_t ph = 0;
    // the current layer's fields, read from the parameter table only when the layer changes
    int64_t lb = 0, lnext = blk[1], Ln = tb.layers[0].n, Lwords = tb.layers[0].words;
    __nv_bfloat16* Lw = reinterpret_cast<__nv_bfloat16*>(tb.layers[0].w);
    int8_t* Lvote = tb.layers[0].vote_out;
    for (int64_t g = blockIdx.x; g < total; g += gridDim.x) {
      if (!bar_wait(bars + 8 * s, ph, abort_flag, budget)) { ok = false; break; }
      if (g >= lnext) {
        while (li + 1 < tb.n_layers && blk[li + 1] <= g) ++li;
        const EwLayer& L = tb.layers[li];
        lb = blk[li]; lnext = blk[li + 1]; Ln = L.n; Lwords = L.words;
        Lw = reinterpret_cast<__nv_bfloat16*>(L.w); Lvote = L.vote_out;
      }
      const int64_t b = g - lb;
      const int ne = (int)min((int64_t)kEntries, Ln - b * kEntries);
      const int nw = (int)min((int64_t)kWords, Lwords - b * kWords);
      const unsigned char* slot = ring + (size_t)s * SB;
      const uint32_t* msg = reinterpret_cast<const uint32_t*>(slot + kWBytes);
      uint32_t c[kPlanes];
#pragma unroll
      for (int p = 0; p < kPlanes; ++p) c[p] = 0u;
      if (j < nw) {
        for (int k0 = 0; k0 < M; k0 += 8) {
          uint32_t x[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) x[i] = (k0 + i < M) ? msg[(k0 + i) * kWords + j] : 0u;
          // the eight words' count per entry (0..8, four planes) by a carry-save tree of full adders
          uint32_t q[4];
          csa_count8(x, q);
          // added into the running count, plane by plane with the carry rippling upward
          uint32_t carry = 0u;
#pragma unroll
          for (int p = 0; p < kPlanes; ++p) {
            const uint32_t a = c[p], bq = p < 4 ? q[p] : 0u;
            c[p] = a ^ bq ^ carry;
            carry = (a & bq) | (carry & (a ^ bq));
          }
        }
      }
      uint32_t gt = 0u, eq = 0xffffffffu;
#pragma unroll
      for (int p = kPlanes - 1; p >= 0; --p) {
        if ((h >> p) & 1) {
          eq &= c[p];
        } else {
          gt |= eq & c[p];
          eq &= ~c[p];
        }
      }
      const uint32_t pos = gt, tie = eq & even;
      const uint32_t plus = tb.tie > 0 ? (pos | tie) : pos;
      const uint32_t zero = zero_ties ? tie : 0u;
      // this warp's 1024 entries of W as four 512-byte rows: lane l takes 16-byte unit 32 q + l (entries
      // 8 (32 q + l) .. + 7), whose vote bits are byte (l & 3) of the word counted by lane 8 q + l / 4
      const int wv = min(max(ne - 1024 * warp, 0), 1024);  // valid entries of the warp (a multiple of 8)
      const uint4* ws = reinterpret_cast<const uint4*>(slot) + 128 * warp;
      uint4* wg = reinterpret_cast<uint4*>(Lw + b * kEntries + 1024 * warp);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int src = 8 * q + (lane >> 2), sh = 8 * (lane & 3);
        const uint32_t pb = __shfl_sync(0xffffffffu, plus, src) >> sh;
        const uint32_t zb = (__shfl_sync(0xffffffffu, zero, src) >> sh) & 0xffu;
        const int u = 32 * q + lane;
        if (8 * u < wv) {
          const uint4 wq = ws[u];
          const uint32_t w4[4] = {wq.x, wq.y, wq.z, wq.w};
          // the eight subtrahends from two table entries (entries 0-3 and 4-7 of the unit)
          const float4 dl = lut[(((pb & 0xfu) | ((zb << 4) & 0xf0u)) << 3) | (lane & 7)];
          const float4 dh = lut[((((pb >> 4) & 0xfu) | (zb & 0xf0u)) << 3) | (lane & 7)];
          const float dv[8] = {dl.x, dl.y, dl.z, dl.w, dh.x, dh.y, dh.z, dh.w};
          uint32_t o[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) {  // entries 2 k (low half) and 2 k + 1 (high half)
            const float d0 = dv[2 * k], d1 = dv[2 * k + 1];
            float r0, r1;
            // both entries' f32 W - d in one two-wide subtraction (round to nearest, per element)
            asm("{\n .reg .b64 a, b, r;\n mov.b64 a, {%2, %3};\n mov.b64 b, {%4, %5};\n"
                " sub.rn.f32x2 r, a, b;\n mov.b64 {%0, %1}, r;\n}"
                : "=f"(r0), "=f"(r1)
                : "f"(__uint_as_float(w4[k] << 16)), "f"(__uint_as_float(w4[k] & 0xffff0000u)), "f"(d0), "f"(d1));
            o[k] = pack_bf16x2_rn(r0, r1);
          }
          wg[u] = make_uint4(o[0], o[1], o[2], o[3]);
        }
      }
      if (Lvote) {  // this lane's own 32 entries, in groups of 8
        const int nent = min(max(ne - 32 * j, 0), 32);
        for (int g8 = 0; g8 < nent / 8; ++g8) {
          const uint32_t pb = pos >> (8 * g8), tbits = tie >> (8 * g8);
          int8_t v8[8];
#pragma unroll
          for (int k = 0; k < 8; ++k) v8[k] = (int8_t)(((pb >> k) & 1u) ? 1 : (((tbits >> k) & 1u) ? tb.tie : -1));
          int8_t* dst = Lvote + b * kEntries + 32 * j + 8 * g8;
          if ((reinterpret_cast<uintptr_t>(dst) & 7) == 0) {
            uint2 pk;
            memcpy(&pk, v8, 8);
            *reinterpret_cast<uint2*>(dst) = pk;
          } else {
#pragma unroll
            for (int k = 0; k < 8; ++k) dst[k] = v8[k];
          }
        }
      }
      __syncwarp();
      if (lane == 0) bar_arrive(bars + 8 * (kSlots + s));  // the warp's reads of the slot are done
      if (++s == kSlots) { s = 0; ph ^= 1u; }
    }
    if (!ok && lane == 0) {
      *abort_flag = 1;
      if (tb.status) atomicOr(tb.status, SMUON_DEV_WAIT_TIMEOUT);
    }
  }
}

// the TMA-staged form takes a launch whose layers all have bf16 W, contiguous and 16-byte aligned, with
// entry counts that are multiples of 8 (whole 16-byte rows of W), and M <= 16
bool bits_tma_eligible(const EwTable& tb) {
  if (tb.src_dtype != SMUON_BITS || tb.M > bitsq::kMaxM || tb.M < 1 || tb.n_layers < 1) return false;
  for (int l = 0; l < tb.n_layers; ++l) {
    const EwLayer& L = tb.layers[l];
    if (!L.w || L.w_dtype != SMUON_BF16 || !L.vec || L.n % 8 != 0 || L.packed_out) return false;
    if (reinterpret_cast<uintptr_t>(L.w) % 16) return false;
    for (int k = 0; k < tb.M; ++k)
      if (reinterpret_cast<uintptr_t>(tb.srcs[L.src_first + k].ptr) % 16) return false;
  }
  return true;
}

template <int kPlanes>
static cudaError_t launch_bits_tma(const EwTable& tb, int sms, cudaStream_t s) {
  const int bytes = bitsq::smem_bytes(tb.M);
  static bool attr_set[256] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 256 && !attr_set[dev]) {
    // the largest form (M = 16) once per device
    cudaError_t e = cudaFuncSetAttribute(k_vote_update_bits_tma<kPlanes>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         bitsq::smem_bytes(bitsq::kMaxM));
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  int64_t blocks = 0;
  for (int l = 0; l < tb.n_layers; ++l) blocks += (tb.layers[l].words + bitsq::kWords - 1) / bitsq::kWords;
  int per_sm = 1;  // as many CTAs as an SM holds with this M's ring
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_vote_update_bits_tma<kPlanes>, bitsq::kThreads, bytes) !=
          cudaSuccess || per_sm < 1)
    per_sm = 1;
  const int grid = (int)std::max<int64_t>(1, std::min<int64_t>(blocks, (int64_t)per_sm * sms));
  k_vote_update_bits_tma<kPlanes><<<grid, bitsq::kThreads, bytes, s>>>(tb);
  return cudaGetLastError();
}

template <int kPlanes>
static void launch_bits(const EwTable& tb, bool has_w, int grid, cudaStream_t s) {
  if (has_w) k_vote_update_bits<true, kPlanes><<<grid, 256, 0, s>>>(tb);
  else k_vote_update_bits<false, kPlanes><<<grid, 256, 0, s>>>(tb);
}

template <bool kPopcount, bool kBf16, typename MaskT>
__global__ void __launch_bounds__(256) k_vote_update(const __grid_constant__ EwTable tb) {
  vote_update_body<kPopcount, kBf16, MaskT>(tb);
}

template <bool kHasW>
__global__ void __launch_bounds__(256, 3) k_vote_update_i8_bf16(const __grid_constant__ EwTable tb) {
  vote_update_int8_bf16<kHasW>(tb);
}

template <bool kHasW>
__global__ void __launch_bounds__(256, 3) k_vote_update_bf16x16(const __grid_constant__ EwTable tb) {
  vote_update_bf16x16<kHasW>(tb);
}

template <bool kHasW>
__global__ void __launch_bounds__(256, 3) k_vote_update_i8src(const __grid_constant__ EwTable tb) {
  vote_update_i8src<kHasW>(tb);
}

cudaError_t launch_vote_update(const EwTable& tb, bool popcount, int grid, int sms, cudaStream_t s) {
  const bool bf = tb.src_dtype == SMUON_BF16;
  // 16 entries per lane, three resident CTAs per SM (launch bounds), one wave
  const int64_t want16 = (tb.total_chunks + 511) / 512;
  const int grid16 = (int)std::max<int64_t>(1, std::min<int64_t>(want16, 3 * sms));
  const bool has_w = tb.layers[0].w != nullptr;  // all layers or none (signs and votes only)
  if (tb.src_dtype == SMUON_BITS && bits_tma_eligible(tb)) {
    if (tb.M <= 15) return launch_bits_tma<4>(tb, sms, s);
    return launch_bits_tma<5>(tb, sms, s);
  }
  if (tb.src_dtype == SMUON_BITS) {
    // one lane per packed word, four resident CTAs per SM, one wave
    const int64_t want = (tb.total_chunks / 4 + 255) / 256;
    const int gridb = (int)std::max<int64_t>(1, std::min<int64_t>(want, 4 * sms));
    if (tb.M <= 15) launch_bits<4>(tb, has_w, gridb, s);
    else if (tb.M <= 31) launch_bits<5>(tb, has_w, gridb, s);
    else launch_bits<7>(tb, has_w, gridb, s);
    return cudaGetLastError();
  }
  if (tb.src_dtype == SMUON_I8) {  // sign matrices: both vote kinds count the same positives
    if (has_w) k_vote_update_i8src<true><<<grid16, 256, 0, s>>>(tb);
    else k_vote_update_i8src<false><<<grid16, 256, 0, s>>>(tb);
    return cudaGetLastError();
  }
  if (bf && (popcount || tb.any_packed) && tb.M <= kMaxWorkers) {
    if (has_w) k_vote_update_bf16x16<true><<<grid16, 256, 0, s>>>(tb);
    else k_vote_update_bf16x16<false><<<grid16, 256, 0, s>>>(tb);
    return cudaGetLastError();
  }
  if (popcount) {
    if (tb.M <= 32) {
      if (bf) k_vote_update<true, true, uint32_t><<<grid, 256, 0, s>>>(tb);
      else k_vote_update<true, false, uint32_t><<<grid, 256, 0, s>>>(tb);
    } else {
      if (bf) k_vote_update<true, true, uint64_t><<<grid, 256, 0, s>>>(tb);
      else k_vote_update<true, false, uint64_t><<<grid, 256, 0, s>>>(tb);
    }
  } else {
    // the packed-counter kernel needs no packed message (it builds none)
    if (bf && !tb.any_packed) {
      if (has_w) k_vote_update_i8_bf16<true><<<grid16, 256, 0, s>>>(tb);
      else k_vote_update_i8_bf16<false><<<grid16, 256, 0, s>>>(tb);
    }
    else if (bf) k_vote_update<false, true, uint32_t><<<grid, 256, 0, s>>>(tb);
    else k_vote_update<false, false, uint32_t><<<grid, 256, 0, s>>>(tb);
  }
  return cudaGetLastError();
}

// SignMuon summary, flow steps 2-3: signs and the 1-bit message only.
__global__ void __launch_bounds__(256) k_sign_pack(const __grid_constant__ EwTable tb,
                                                   uint32_t* packed, int8_t* signs) {
  const int lane = threadIdx.x & 31;
  const int64_t warp_global = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t warps_total = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const EwLayer& L = tb.layers[0];
  for (int64_t wbase = warp_global * 32; wbase < tb.total_chunks; wbase += warps_total * 32) {
    const int64_t chunk = wbase + lane;
    const bool active = chunk < tb.total_chunks;
    const int64_t e0 = chunk * 8;
    const bool live = active && e0 < L.n;
    for (int wk = 0; wk < tb.M; ++wk) {
      const EwSrc& S = tb.srcs[wk];
      float u[8];
      if (live) load8(S.ptr, S.ld, tb.src_dtype, L, e0, L.vec, u);
      uint32_t byte = 0;
      int8_t sg[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const bool pos = live && (e0 + k < L.n) && (u[k] >= 0.f);
        byte |= (uint32_t)pos << k;
        sg[k] = pos ? 1 : -1;
      }
      if (packed) {
        const uint32_t word = gather_word(byte, lane);
        if (active && (lane & 3) == 0) packed[(int64_t)wk * L.words + (chunk >> 2)] = word;
      }
      if (signs && live) {
        int8_t* dst = signs + (int64_t)wk * L.n + e0;
        if (e0 + 8 <= L.n && ((reinterpret_cast<uintptr_t>(dst) & 7) == 0)) {
          uint2 pk;
          memcpy(&pk, sg, 8);
          *reinterpret_cast<uint2*>(dst) = pk;
        } else {
          for (int k = 0; k < 8; ++k) if (e0 + k < L.n) dst[k] = sg[k];
        }
      }
    }
  }
}

// SignMuon summary, flow steps 3-4: vote from the all-gathered bits (sum =
// 2*popcount - M) or from the all-reduced int8 signs. One thread per 32
// entries (one packed word per worker).
__global__ void __launch_bounds__(256) k_vote(const uint32_t* packed, const int8_t* signs, int M,
                                              int64_t N, int64_t words, int tie, int8_t* vote) {
  const int64_t nw = (N + 31) / 32;
  for (int64_t w = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; w < nw;
       w += (int64_t)gridDim.x * blockDim.x) {
    const int64_t e0 = w * 32;
    const int nvalid = (N - e0) < 32 ? (int)(N - e0) : 32;
    int8_t out[32];
    if (packed) {
      uint32_t bits[kMaxWorkers];
      for (int k = 0; k < M; ++k) bits[k] = packed[(int64_t)k * words + w];
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        uint64_t mask = 0;
        for (int k = 0; k < M; ++k) mask |= (uint64_t)((bits[k] >> j) & 1u) << k;
        out[j] = threshold(2 * __popcll(mask) - M, tie);
      }
    } else {
      int sum[32];  // rows may be partial sums (an all-reduced message): add in int
#pragma unroll
      for (int j = 0; j < 32; ++j) sum[j] = 0;
      for (int k = 0; k < M; ++k) {
        const int8_t* src = signs + (int64_t)k * N + e0;
#pragma unroll
        for (int j = 0; j < 32; ++j) if (j < nvalid) sum[j] += src[j];
      }
#pragma unroll
      for (int j = 0; j < 32; ++j) out[j] = threshold(sum[j], tie);
    }
    if (nvalid == 32 && ((reinterpret_cast<uintptr_t>(vote + e0) & 15) == 0)) {
      uint4 a, b;
      memcpy(&a, out, 16);
      memcpy(&b, out + 16, 16);
      reinterpret_cast<uint4*>(vote + e0)[0] = a;
      reinterpret_cast<uint4*>(vote + e0)[1] = b;
    } else {
      for (int j = 0; j < nvalid; ++j) vote[e0 + j] = out[j];
    }
  }
}

// W <- W - eta * v (vote, exact product) or W - f32(eta * D) (dense), reading R9.
__global__ void __launch_bounds__(256) k_update_src(const __grid_constant__ EwTable tb) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t chunk = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; chunk < tb.total_chunks;
       chunk += stride) {
    const int li = find_layer(&tb, chunk);
    const EwLayer& L = tb.layers[li];
    const int64_t e0 = (chunk - L.chunk_begin) * 8;
    if (e0 >= L.n) continue;
    const EwSrc& S = tb.srcs[L.src_first];
    float d[8], w[8];
    load8(S.ptr, S.ld, tb.src_dtype, L, e0, L.vec, d);
    load8(L.w, L.w_ld, L.w_dtype, L, e0, L.vec, w);
#pragma unroll
    for (int k = 0; k < 8; ++k) w[k] = __fsub_rn(w[k], __fmul_rn(tb.eta, d[k]));
    store8(L.w, L.w_ld, L.w_dtype, L, e0, L.vec, w);
  }
}

// LionMuon summary, methodology items 1-2, sign step: per worker
// G_hat = f32(beta1*M) + f32((1-beta1)*G), bit = G_hat >= 0, then
// EMA M <- f32(beta2*M) + f32((1-beta2)*G); majority vote; W update.
__global__ void __launch_bounds__(256) k_lion_sign(const __grid_constant__ EwTable tb) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t chunk = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; chunk < tb.total_chunks;
       chunk += stride) {
    const int li = find_layer(&tb, chunk);
    const EwLayer& L = tb.layers[li];
    const int64_t e0 = (chunk - L.chunk_begin) * 8;
    if (e0 >= L.n) continue;
    uint64_t mask[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) mask[k] = 0;
    for (int wk0 = 0; wk0 < tb.M; wk0 += 2) {
      float mo[2][8], gr[2][8];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int wk = wk0 + j;
        if (wk < tb.M) {
          load8(tb.srcs[L.src_first + 2 * wk].ptr, tb.srcs[L.src_first + 2 * wk].ld, SMUON_F32, L, e0, L.vec, mo[j]);
          if (tb.gen_on)
            crng::gaussian8(tb.gen_seed + (uint32_t)wk, L.key1, tb.gen_step, e0, tb.gen_sigma, gr[j]);
          else
            load8(tb.srcs[L.src_first + 2 * wk + 1].ptr, tb.srcs[L.src_first + 2 * wk + 1].ld, SMUON_F32, L, e0,
                  L.vec, gr[j]);
        }
      }
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int wk = wk0 + j;
        if (wk >= tb.M) break;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const float gh = __fadd_rn(__fmul_rn(tb.beta1, mo[j][k]), __fmul_rn(tb.c1, gr[j][k]));
          mask[k] |= (uint64_t)(gh >= 0.f) << wk;
          mo[j][k] = __fadd_rn(__fmul_rn(tb.beta2, mo[j][k]), __fmul_rn(tb.c2, gr[j][k]));
        }
        const EwSrc& S = tb.srcs[L.src_first + 2 * wk];  // EMA (f32, in/out)
        store8(const_cast<void*>(S.ptr), S.ld, SMUON_F32, L, e0, L.vec, mo[j]);
      }
    }
    float w[8];
    load8(L.w, L.w_ld, L.w_dtype, L, e0, L.vec, w);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int8_t v = threshold(2 * __popcll(mask[k]) - tb.M, tb.tie);
      w[k] = __fsub_rn(w[k], tb.eta * (float)v);
    }
    store8(L.w, L.w_ld, L.w_dtype, L, e0, L.vec, w);
  }
}

// LionMuon Muon step prologue (reading R11): mean over workers of G_hat into a
// contiguous f32 buffer, and the EMA update of every worker. With ghat_out (the
// vote reading of the Muon step) every worker's G_hat is written instead, to
// the contiguous f32 block aux + k * n.
__global__ void __launch_bounds__(256) k_lion_mean(const __grid_constant__ EwTable tb) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  const float invM = 1.f / (float)tb.M;
  for (int64_t chunk = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; chunk < tb.total_chunks;
       chunk += stride) {
    const int li = find_layer(&tb, chunk);
    const EwLayer& L = tb.layers[li];
    const int64_t e0 = (chunk - L.chunk_begin) * 8;
    if (e0 >= L.n) continue;
    float acc[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) acc[k] = 0.f;
    for (int wk = 0; wk < tb.M; ++wk) {
      const EwSrc& S = tb.srcs[L.src_first + 2 * wk];
      const EwSrc& Gs = tb.srcs[L.src_first + 2 * wk + 1];
      float mo[8], gr[8];
      load8(S.ptr, S.ld, SMUON_F32, L, e0, L.vec, mo);
      if (tb.gen_on)
        crng::gaussian8(tb.gen_seed + (uint32_t)wk, L.key1, tb.gen_step, e0, tb.gen_sigma, gr);
      else
        load8(Gs.ptr, Gs.ld, SMUON_F32, L, e0, L.vec, gr);
      float gh[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        gh[k] = __fadd_rn(__fmul_rn(tb.beta1, mo[k]), __fmul_rn(tb.c1, gr[k]));
        acc[k] = __fadd_rn(acc[k], gh[k]);
        mo[k] = __fadd_rn(__fmul_rn(tb.beta2, mo[k]), __fmul_rn(tb.c2, gr[k]));
      }
      store8(const_cast<void*>(S.ptr), S.ld, SMUON_F32, L, e0, L.vec, mo);
      if (tb.ghat_out) store8(reinterpret_cast<float*>(L.aux) + (int64_t)wk * L.n, L.cols, SMUON_F32, L, e0, L.vec_aux, gh);
    }
    if (tb.ghat_out) continue;
#pragma unroll
    for (int k = 0; k < 8; ++k) acc[k] = __fmul_rn(acc[k], invM);
    // the mean buffer is contiguous (ld == cols) f32 in the workspace
    store8(L.aux, L.cols, SMUON_F32, L, e0, L.vec_aux, acc);
  }
}

// CacheMuon summary, method item 3: err = sqrt(sum of squared residuals)/sqrt(m),
// accept iff err <= gamma (NaN rejects), counters updated on the device.
__global__ void k_probe_finalize(const Plan* plan) {
  const PlanHeader& h = plan->h;
  if (threadIdx.x >= 32) return;
  const int lane = threadIdx.x;
  const int n = kProbeSlots * h.total_tiles[ST_PROBE];
  float acc = 0.f;
  for (int i = lane; i < n; i += 32) acc += h.probe_partials[i];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) {
    const int m = h.groups[0].m;
    const float err = sqrtf(acc) / sqrtf((float)m);
    const int accept = (err <= h.gamma) ? 1 : 0;  // NaN compares false
    *h.d_err = err;
    *h.d_accept = accept;
    if (h.counters) {
      h.counters->probes += 1;
      if (accept) h.counters->hits += 1; else h.counters->misses += 1;
    }
  }
}

// First CacheMuon step (no cached transform): reject without a probe.
__global__ void k_probe_nocache(float* d_err, int32_t* d_accept, cachemuon_counters* counters) {
  *d_err = __int_as_float(0x7f800000);
  *d_accept = 0;
  if (counters) counters->misses += 1;
}

// Harness: sigma * N(0, 1) from the counter-based stream of each matrix
// (key words per matrix, counter word 2 = the step), written as float32.
__global__ void __launch_bounds__(256) k_harness_gaussian(const __grid_constant__ EwTable tb) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t chunk = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; chunk < tb.total_chunks;
       chunk += stride) {
    const int li = find_layer(&tb, chunk);
    const EwLayer& L = tb.layers[li];
    const int64_t e0 = (chunk - L.chunk_begin) * 8;
    if (e0 >= L.n) continue;
    float v[8];
    crng::gaussian8(L.key0, L.key1, tb.gen_step, e0, tb.gen_sigma, v);
    store8(L.w, L.w_ld, SMUON_F32, L, e0, L.vec, v);
  }
}

}  // namespace smuon
