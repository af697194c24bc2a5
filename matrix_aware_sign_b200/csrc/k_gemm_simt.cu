// k_gemm_simt.cu -- grouped Newton-Schulz GEMM stages on CUDA cores.
//
// Used for the FP32 reference mode (float32 operands, float32 FMA) and as a
// diagnostic BF16-operand variant that the tcgen05 kernel is checked against.
// Tile 64 x 64 x 16, 256 threads, 4 x 4 outputs per thread; persistent CTAs
// walk the plan's tile list of one stage.
#include "epilogue.cuh"

namespace smuon {

template <typename T>
__device__ __forceinline__ float to_f(T v);
template <>
__device__ __forceinline__ float to_f<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }

// Operands of stage st: A is K-major (row-major [Mo][K]); B is either
// N x K row-major (kNT, the Gram forms) or K x N row-major (NN, B X and B Q).
struct SimtOps {
  const void* A;
  int64_t lda;
  const void* B;
  int64_t ldb;
  int nt;
  int K;
};

__device__ __forceinline__ SimtOps simt_ops(const TileCtx& t, int iter) {
  const GroupDesc& g = *t.g;
  const int m = g.m;
  SimtOps o;
  const int esz = t.bf ? 2 : 4;
  auto at = [&](const void* base, int64_t ld) {
    return reinterpret_cast<const void*>(reinterpret_cast<const char*>(base) + (int64_t)t.z * m * ld * esz);
  };
  switch (t.stage) {
    case ST_GRAM:
      o.A = at(g.xop[iter & 1], g.ldn); o.lda = g.ldn;
      o.B = o.A; o.ldb = g.ldn; o.nt = 1; o.K = g.n; break;
    case ST_POLY:
      o.A = at(g.aop, g.ldm); o.lda = g.ldm;
      o.B = o.A; o.ldb = g.ldm; o.nt = 1; o.K = m; break;
    case ST_AXPY:
      o.A = at(g.bop, g.ldm); o.lda = g.ldm;
      o.B = at(g.xop[iter & 1], g.ldn); o.ldb = g.ldn; o.nt = 0; o.K = m; break;
    case ST_QAXPY:
      o.A = at(g.bop, g.ldm); o.lda = g.ldm;
      o.B = at(g.qop[iter & 1], g.ldm); o.ldb = g.ldm; o.nt = 0; o.K = m; break;
    case ST_REUSE:
      o.A = t.md->q_ptr; o.lda = t.md->q_ld;   // user Q (bf16)
      o.B = at(g.xop[0], g.ldn); o.ldb = g.ldn; o.nt = 0; o.K = m; break;
    default:  // ST_PROBE
      o.A = at(g.xop[1], g.ldn); o.lda = g.ldn;
      o.B = o.A; o.ldb = g.ldn; o.nt = 1; o.K = g.n; break;
  }
  return o;
}

template <typename TOp>
__device__ __forceinline__ void gemm_simt_body(const Plan* plan, int stage, int iter) {
  const PlanHeader& h = plan->h;
  __shared__ float As[16][64 + 4];
  __shared__ float Bs[16][64 + 4];
  __shared__ float red[8];
  const int tid = threadIdx.x;
  const int tx = tid & 15, ty = tid >> 4;
  const int total = h.total_tiles[stage];
  for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
    int tm, tn;
    TileCtx t = make_ctx(h, stage, iter, tile, tm, tn);
    const SimtOps o = simt_ops(t, iter);
    const TOp* A = reinterpret_cast<const TOp*>(o.A);
    const TOp* B = reinterpret_cast<const TOp*>(o.B);
    const int row0 = tm * 64, col0 = tn * 64;
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
    for (int k0 = 0; k0 < o.K; k0 += 16) {
      // A tile: 64 rows x 16 k; thread loads 4 elements
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int e = tid + q * 256;
        const int r = e >> 4, kk = e & 15;
        const int gr = row0 + r, gk = k0 + kk;
        As[kk][r] = (gr < t.Mo && gk < o.K) ? to_f<TOp>(A[(int64_t)gr * o.lda + gk]) : 0.f;
      }
      if (o.nt) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int e = tid + q * 256;
          const int r = e >> 4, kk = e & 15;
          const int gn = col0 + r, gk = k0 + kk;
          Bs[kk][r] = (gn < t.No && gk < o.K) ? to_f<TOp>(B[(int64_t)gn * o.ldb + gk]) : 0.f;
        }
      } else {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int e = tid + q * 256;
          const int kk = e >> 6, c = e & 63;
          const int gn = col0 + c, gk = k0 + kk;
          Bs[kk][c] = (gn < t.No && gk < o.K) ? to_f<TOp>(B[(int64_t)gk * o.ldb + gn]) : 0.f;
        }
      }
      __syncthreads();
#pragma unroll
      for (int kk = 0; kk < 16; ++kk) {
        float a[4], b[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
        for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx * 4 + j];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
      }
      __syncthreads();
    }
    float pacc = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) epi_chunk<4>(t, row0 + ty * 4 + i, col0 + tx * 4, acc[i], &pacc);
    if (stage == ST_PROBE) {
#pragma unroll
      for (int o2 = 16; o2 > 0; o2 >>= 1) pacc += __shfl_xor_sync(0xffffffffu, pacc, o2);
      if ((tid & 31) == 0) red[tid >> 5] = pacc;
      __syncthreads();
      if (tid == 0) {
        float s = 0.f;
#pragma unroll
        for (int w = 0; w < 8; ++w) s += red[w];
        h.probe_partials[kProbeSlots * tile] = s;
        for (int q = 1; q < kProbeSlots; ++q) h.probe_partials[kProbeSlots * tile + q] = 0.f;
      }
      __syncthreads();
    }
  }
}

__global__ void __launch_bounds__(256) k_gemm_simt_f32(const Plan* plan, int stage, int iter,
                                                       const int32_t* skip) {
  if (skip && *skip) return;
  gemm_simt_body<float>(plan, stage, iter);
}
__global__ void __launch_bounds__(256) k_gemm_simt_bf16(const Plan* plan, int stage, int iter,
                                                        const int32_t* skip) {
  if (skip && *skip) return;
  gemm_simt_body<__nv_bfloat16>(plan, stage, iter);
}

}  // namespace smuon
