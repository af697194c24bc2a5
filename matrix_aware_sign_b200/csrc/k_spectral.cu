// k_spectral.cu -- spectral-norm normalisation of the Newton-Schulz input.
//
// The "SignMuon" summary (section 4) allows the spectral norm in place of the
// Frobenius norm. The first Gram stage already holds A_0 = s^2 X X^T (s the
// Frobenius scale), whose largest eigenvalue is (s ||M||_2)^2. A Lanczos
// iteration with full reorthogonalisation estimates it for every matrix of
// the batch at once; the first step's epilogues then rescale by
// r = 1 / (sqrt(lambda_max) + eps s), so that X_0 = s r M = M / (||M||_2 + eps).
//
// Per Lanczos step j: w = A v_j for the matrices still iterating
// (k_lz_matvec: one warp per row, their rows spread evenly; the list comes
// from the previous step's last block, or k_lz_compact before the first),
// then w is orthogonalised against v_0 .. v_j by classical Gram-Schmidt done
// twice (one warp per basis vector for the coefficients); alpha_j is the v_j
// coefficient of the two passes together, beta_j = ||w|| and
// v_{j+1} = w / beta_j (k_lz_step: one CTA per matrix). In exact arithmetic the
// coefficients of v_0 .. v_{j-2} vanish and that of v_{j-1} is beta_{j-1}, the
// three-term recurrence; the full passes keep the basis orthogonal in float32.
// Every fourth step the largest Ritz value theta of the tridiagonal (alpha,
// beta) matrix and its eigenvector y are formed; a matrix stops when the
// residual beta_j |y_last|, which bounds |lambda - theta|, is below 1e-4 theta
// (its later launches skip it), and at the latest after kLanczosSteps steps.
// (the error itself is near r^2 / gap, far smaller: below 1e-7 on random
// Gaussian matrices of the workload shapes, which stop after 16 to 56 steps).
// k_lz_finish then takes lambda_max of the tridiagonal matrix by bisection on
// its Sturm counts. Vectors are stored with a stride of m rounded up to 4
// floats, so rows of A and vectors load as float4.
#include "kernels.cuh"

namespace smuon {

namespace {

__device__ __forceinline__ float* lz_vec(const PlanHeader& h, const MatDesc& md, int j) {
  const GroupDesc& g = h.groups[md.group];
  return h.lz + md.lz_off + (int64_t)j * lz_stride(g.m);
}

// block-wide sum (256 threads); every thread gets the result
__device__ __forceinline__ float block_sum(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  float t = 0.f;
  if (l < (int)(blockDim.x >> 5)) t = red[l];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
  return t;
}

// Sturm count: eigenvalues of the k x k tridiagonal matrix (a, b) below x,
// b[i] coupling rows i and i + 1 (float32: the count is exact for a matrix
// within a few ulps of T, which bounds the bisection's error near 1e-7 of ||T||)
__device__ __forceinline__ int sturm_below(const float* a, const float* b, int k, float x) {
  int count = 0;
  float d = 1.f;
  for (int i = 0; i < k; ++i) {
    const float b2 = i > 0 ? b[i - 1] * b[i - 1] : 0.f;
    d = (a[i] - x) - (i > 0 ? __fdiv_rn(b2, d) : 0.f);
    if (d == 0.f) d = -1e-30f;
    if (d < 0.f) ++count;
  }
  return count;
}

// largest eigenvalue of (a, b), called by all 32 lanes of a warp: each round
// the lanes take Sturm counts at 32 interior points of the Gershgorin interval
// [lo, hi] and it shrinks to the gap where the count reaches k (33x per round)
__device__ __forceinline__ float tri_lambda_max(const float* a, const float* b, int k, int lane) {
  float lo = 0.f, hi = 0.f;  // lo <= 0: A_0 is positive semidefinite
  for (int t = 0; t < k; ++t) {
    const float rad = (t > 0 ? fabsf(b[t - 1]) : 0.f) + (t + 1 < k ? fabsf(b[t]) : 0.f);
    hi = fmaxf(hi, a[t] + rad);
    lo = fminf(lo, a[t] - rad);
  }
  for (int round = 0; round < 8 && hi - lo > 2e-7f * fmaxf(fabsf(hi), 1e-30f); ++round) {
    const float x = lo + (hi - lo) * (float)(lane + 1) * (1.f / 33.f);
    const unsigned above = __ballot_sync(0xffffffffu, sturm_below(a, b, k, x) == k);
    if (above) {  // lowest point with every eigenvalue below it
      const int f = __ffs(above) - 1;
      const float nhi = lo + (hi - lo) * (float)(f + 1) * (1.f / 33.f);
      lo = f > 0 ? lo + (hi - lo) * (float)f * (1.f / 33.f) : lo;
      hi = nhi;
    } else {
      lo = lo + (hi - lo) * (32.f / 33.f);
    }
  }
  return hi;
}

// |last component| of the unit eigenvector of (a, b) for its largest
// eigenvalue theta, by the recurrence of the rows run backward from
// y_{k-1} = 1. The eigenvector of a converged Ritz value decays toward its
// last index, so backward is the direction in which it grows: the stable one
// (forward, the tiny last component would come out of a cancellation that
// theta's own rounding swamps). A running rescale keeps the values finite.
__device__ __forceinline__ float tri_last_component(const float* a, const float* b, int k, float theta) {
  float y1 = 0.f, y = 1.f, last = 1.f, nrm = 1.f;  // y = y_i, y1 = y_{i+1}
  for (int i = k - 1; i >= 1; --i) {
    const float ym = ((theta - a[i]) * y - (i + 1 < k ? b[i] * y1 : 0.f)) / b[i - 1];
    y1 = y;
    y = ym;
    nrm += ym * ym;
    if (nrm > 1e30f) { y *= 1e-15f; y1 *= 1e-15f; last *= 1e-15f; nrm *= 1e-30f; }
  }
  return last * rsqrtf(nrm);
}

}  // namespace

// v_0: a fixed vector with entries in [0.5, 1.5) from an integer hash, normalised
__global__ void __launch_bounds__(256) k_lz_start(const Plan* plan, const int32_t* skip) {
  if (skip && *skip) return;
  const PlanHeader& h = plan->h;
  __shared__ float red[8];
  for (int i = blockIdx.x; i < h.n_mats; i += gridDim.x) {
    const MatDesc& md = h.mats[i];
    const int m = h.groups[md.group].m;
    float* v = lz_vec(h, md, 0);
    float ss = 0.f;
    for (int k = threadIdx.x; k < m; k += blockDim.x) {
      const uint32_t x = (uint32_t)k * 0x9E3779B1u + 0x7F4A7C15u;
      const float e = 0.5f + (float)((x >> 8) & 0xFFFFu) * (1.f / 65536.f);
      v[k] = e;
      ss += e * e;
    }
    const float inv = rsqrtf(block_sum(ss, red));
    for (int k = threadIdx.x; k < m; k += blockDim.x) v[k] *= inv;
    __syncthreads();
  }
}

// w = A v_j for every matrix: one warp per row of A, each warp over a
// contiguous range of the flattened rows (one matrix lookup per range). A is
// the f32 A_0, or in the plain BF16 modes with c != 0 the bf16 operand copy
// of it: half the bytes, for a relative perturbation of lambda_max near
// 2^-9 / sqrt(m), inside those modes' own rounding. The split mode keeps the
// f32 A_0: its sign criterion is tight enough to notice that perturbation.
__global__ void __launch_bounds__(256) k_lz_matvec(const Plan* plan, int j, const int32_t* skip) {
  if (skip && *skip) return;
  const PlanHeader& h = plan->h;
  const int lane = threadIdx.x & 31;
  const int n_act = h.lz_act[0];
  const int32_t* act_rows = h.lz_act + 1;              // [n_act + 1] prefix of the active matrices' rows
  const int32_t* act_mat = h.lz_act + 2 + h.n_mats;    // [n_act] their indices
  const int64_t warps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t total = n_act > 0 ? act_rows[n_act] : 0;
  const int64_t per = (total + warps - 1) / warps;
  int64_t row = warp * per;
  const int64_t end = min(total, row + per);
  if (row >= end) return;
  const bool use_bf = h.mode != MODE_SIMT_F32 && h.c != 0.f && !(h.flags & SMUON_NS_SPLIT_BF16);
  int q;  // active entry holding `row`: the last with act_rows[q] <= row
  {
    int lo = 0, hi = n_act - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (act_rows[mid] <= row) lo = mid; else hi = mid - 1;
    }
    q = lo;
  }
  while (row < end) {
    const int i = act_mat[q];
    const MatDesc& md = h.mats[i];
    const GroupDesc& g = h.groups[md.group];
    const int m = g.m;
    const int64_t ldm = g.ldm;
    const int64_t r_first = act_rows[q];
    const int64_t r_stop = min(end, (int64_t)act_rows[q + 1]);
    const float* __restrict__ v = h.lz + md.lz_off + (int64_t)j * lz_stride(m);  // 16-byte aligned
    float* __restrict__ w = h.lz + md.lz_off + (int64_t)(kLanczosSteps + 1) * lz_stride(m);
    const float* af = g.af + (int64_t)md.z * m * ldm;
    const __nv_bfloat16* ab = reinterpret_cast<const __nv_bfloat16*>(g.aop) + (int64_t)md.z * m * ldm;
    for (; row < r_stop; ++row) {
      const int r = (int)(row - r_first);
      float acc = 0.f;
      if (use_bf) {  // rows 256-byte aligned (ldm % 128 == 0): 8 bf16 per 16-byte load
        const uint4* a = reinterpret_cast<const uint4*>(ab + (int64_t)r * ldm);
        const int m8 = m >> 3;
        for (int k = lane; k < m8; k += 32) {
          const uint4 x = a[k];
          const float4 y0 = reinterpret_cast<const float4*>(v)[2 * k];
          const float4 y1 = reinterpret_cast<const float4*>(v)[2 * k + 1];
          acc += __uint_as_float(x.x << 16) * y0.x + __uint_as_float(x.x & 0xffff0000u) * y0.y +
                 __uint_as_float(x.y << 16) * y0.z + __uint_as_float(x.y & 0xffff0000u) * y0.w +
                 __uint_as_float(x.z << 16) * y1.x + __uint_as_float(x.z & 0xffff0000u) * y1.y +
                 __uint_as_float(x.w << 16) * y1.z + __uint_as_float(x.w & 0xffff0000u) * y1.w;
        }
        for (int k = 8 * m8 + lane; k < m; k += 32) acc += __bfloat162float(ab[(int64_t)r * ldm + k]) * v[k];
      } else {  // rows 512-byte aligned
        const float* a = af + (int64_t)r * ldm;
        const int m4 = m >> 2;
        for (int k = lane; k < m4; k += 32) {
          const float4 x = reinterpret_cast<const float4*>(a)[k];
          const float4 y = reinterpret_cast<const float4*>(v)[k];
          acc += x.x * y.x + x.y * y.y + x.z * y.z + x.w * y.w;
        }
        for (int k = 4 * m4 + lane; k < m; k += 32) acc += a[k] * v[k];
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      if (lane == 0) w[r] = acc;
    }
    ++q;
  }
}

// the matrices still iterating after step j (all of them for j < 0: before
// the first step), written into h.lz_act by the calling block (a multiple of
// 32 threads, up to 1024; up to 4096 matrices): a matrix continues while its
// last beta is nonzero. The betas come from other blocks of the same launch
// when the last block of k_lz_step calls this, so they are read past L1.
__device__ void lz_compact_block(const PlanHeader& h, int j) {
  const int n = h.n_mats;
  const int per = (n + (int)blockDim.x - 1) / (int)blockDim.x;
  const int first = (int)threadIdx.x * per;
  auto active = [&](int i) {
    return j < 0 || __ldcg(h.lz_ab + (int64_t)i * 2 * kLanczosSteps + kLanczosSteps + j) != 0.f;
  };
  int cnt = 0, rows = 0;
  for (int i = first; i < min(n, first + per); ++i)
    if (active(i)) { ++cnt; rows += h.lz_rows[i + 1] - h.lz_rows[i]; }
  // block-wide exclusive scan of (cnt, rows)
  __shared__ int s_cnt[32], s_rows[32];
  const int lane = threadIdx.x & 31, wi = threadIdx.x >> 5, nw = (int)(blockDim.x >> 5);
  int ic = cnt, ir = rows;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int c = __shfl_up_sync(0xffffffffu, ic, o), r = __shfl_up_sync(0xffffffffu, ir, o);
    if (lane >= o) { ic += c; ir += r; }
  }
  if (lane == 31) { s_cnt[wi] = ic; s_rows[wi] = ir; }
  __syncthreads();
  if (wi == 0) {
    int c = lane < nw ? s_cnt[lane] : 0, r = lane < nw ? s_rows[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int c2 = __shfl_up_sync(0xffffffffu, c, o), r2 = __shfl_up_sync(0xffffffffu, r, o);
      if (lane >= o) { c += c2; r += r2; }
    }
    s_cnt[lane] = c;  // inclusive over warps
    s_rows[lane] = r;
  }
  __syncthreads();
  int pc = ic - cnt + (wi > 0 ? s_cnt[wi - 1] : 0);  // exclusive prefix of this thread
  int pr = ir - rows + (wi > 0 ? s_rows[wi - 1] : 0);
  int32_t* act_rows = h.lz_act + 1;
  int32_t* act_mat = h.lz_act + 2 + n;
  for (int i = first; i < min(n, first + per); ++i)
    if (active(i)) {
      act_mat[pc] = i;
      act_rows[pc] = pr;
      ++pc;
      pr += h.lz_rows[i + 1] - h.lz_rows[i];
    }
  if (threadIdx.x == blockDim.x - 1) {  // the last thread ends with the totals
    h.lz_act[0] = pc;
    act_rows[pc] = pr;
  }
  __syncthreads();
}

// the first active list (every matrix) and a zero ticket for the step launches;
// later lists come from the last block of each k_lz_step launch
__global__ void __launch_bounds__(1024) k_lz_compact(const Plan* plan, int j, const int32_t* skip) {
  if (skip && *skip) return;
  const PlanHeader& h = plan->h;
  lz_compact_block(h, j);
  if (threadIdx.x == 0) h.lz_act[2 * h.n_mats + 2] = 0;
}

// one classical Gram-Schmidt pass of w against v_0 .. v_j: the coefficients
// by one warp per basis vector, then w -= sum_t c_t v_t; returns c_j
__device__ __forceinline__ float cgs_pass(const float* __restrict__ V, int64_t st, int m, int j,
                                          float* __restrict__ w, float* coef) {
  const int wi = threadIdx.x >> 5, l = threadIdx.x & 31, nw = blockDim.x >> 5;
  const int m4 = m >> 2;
  for (int t = wi; t <= j; t += nw) {
    const float* vt = V + t * st;  // 16-byte aligned, as w
    float d = 0.f;
    for (int k = l; k < m4; k += 32) {
      const float4 x = reinterpret_cast<const float4*>(w)[k];
      const float4 y = reinterpret_cast<const float4*>(vt)[k];
      d += x.x * y.x + x.y * y.y + x.z * y.z + x.w * y.w;
    }
    for (int k = 4 * m4 + l; k < m; k += 32) d += w[k] * vt[k];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) d += __shfl_xor_sync(0xffffffffu, d, o);
    if (l == 0) coef[t] = d;
  }
  __syncthreads();
  for (int k = threadIdx.x; k < m; k += blockDim.x) {
    float wk = w[k];
    for (int t = 0; t <= j; ++t) wk -= coef[t] * V[t * st + k];
    w[k] = wk;
  }
  const float cj = coef[j];
  __syncthreads();  // coef is rewritten by the next pass, w read across threads
  return cj;
}

// one Lanczos step per matrix (one CTA of 256 threads each)
__global__ void __launch_bounds__(256) k_lz_step(const Plan* plan, int j, const int32_t* skip) {
  if (skip && *skip) return;
  const PlanHeader& h = plan->h;
  __shared__ float coef[kLanczosSteps];
  __shared__ float red1[8];
  __shared__ float ta[kLanczosSteps], tb[kLanczosSteps];
  __shared__ int s_done;
  for (int i = blockIdx.x; i < h.n_mats; i += gridDim.x) {
    const MatDesc& md = h.mats[i];
    const int m = h.groups[md.group].m;
    float* ab = h.lz_ab + (int64_t)i * 2 * kLanczosSteps;  // alpha[0..K), beta[K..2K)
    if (j > 0 && ab[kLanczosSteps + j - 1] == 0.f) {  // stopped earlier (converged or broke down)
      if (threadIdx.x == 0) { ab[j] = 0.f; ab[kLanczosSteps + j] = 0.f; }
      continue;
    }
    const int64_t st = lz_stride(m);
    float* V = h.lz + md.lz_off;  // v_0 .. v_K, then w
    float* w = V + (int64_t)(kLanczosSteps + 1) * st;
    const float a1 = cgs_pass(V, st, m, j, w, coef);
    const float alpha = a1 + cgs_pass(V, st, m, j, w, coef);
    float ss = 0.f;
    for (int k = threadIdx.x; k < m; k += blockDim.x) ss += w[k] * w[k];
    const float beta = sqrtf(block_sum(ss, red1));  // the same value in every thread
    bool ok = beta > 1e-6f * fabsf(alpha) && beta > 1e-30f && j + 1 < kLanczosSteps;
    if (ok && j >= 11 && (j & 3) == 3) {  // converged? residual of the largest Ritz pair
      if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        for (int t = lane; t <= j; t += 32) {
          ta[t] = t < j ? ab[t] : alpha;
          tb[t] = t < j ? ab[kLanczosSteps + t] : 0.f;
        }
        __syncwarp();
        const float theta = tri_lambda_max(ta, tb, j + 1, lane);
        if (lane == 0) s_done = beta * tri_last_component(ta, tb, j + 1, theta) <= 1e-4f * theta ? 1 : 0;
      }
      __syncthreads();
      if (s_done) ok = false;  // the (alpha, beta) so far hold lambda_max
    }
    if (ok) {
      float* vn = V + (int64_t)(j + 1) * st;
      const float inv = 1.f / beta;
      for (int k = threadIdx.x; k < m; k += blockDim.x) vn[k] = w[k] * inv;
    }
    if (threadIdx.x == 0) { ab[j] = alpha; ab[kLanczosSteps + j] = ok ? beta : 0.f; }
    __syncthreads();
  }
  // the last block to finish lists the matrices still iterating for the next A v launch (no block waits:
  // the ticket only tells the last one that every other block's betas are written and fenced)
  __shared__ int s_last;
  if (threadIdx.x == 0) {
    __threadfence();
    s_last = atomicAdd(h.lz_act + 2 * h.n_mats + 2, 1) == (int)gridDim.x - 1;
  }
  __syncthreads();
  if (s_last) {
    __threadfence();
    lz_compact_block(h, j);
    if (threadIdx.x == 0) h.lz_act[2 * h.n_mats + 2] = 0;  // ready for the next step's launch
  }
}

// lambda_max of each matrix's tridiagonal matrix, one warp per matrix, then
// r = 1 / (sqrt(lambda) + eps s)
__global__ void __launch_bounds__(256) k_lz_finish(const Plan* plan, const int32_t* skip) {
  if (skip && *skip) return;
  const PlanHeader& h = plan->h;
  __shared__ float fa[8][kLanczosSteps], fb[8][kLanczosSteps];
  const int lane = threadIdx.x & 31, wi = threadIdx.x >> 5;
  const int i = (int)((blockIdx.x * blockDim.x + threadIdx.x) >> 5);
  if (i >= h.n_mats) return;
  const float* alpha = h.lz_ab + (int64_t)i * 2 * kLanczosSteps;
  const float* beta = alpha + kLanczosSteps;
  int k = 1;  // the Krylov dimension actually built: steps up to the first stop
  while (k < kLanczosSteps && beta[k - 1] != 0.f) ++k;
  for (int t = lane; t < k; t += 32) {
    fa[wi][t] = alpha[t];
    fb[wi][t] = t + 1 < k ? beta[t] : 0.f;
  }
  __syncwarp();
  const float lam = tri_lambda_max(fa[wi], fb[wi], k, lane);  // 0 for a zero matrix: s r = 1/eps then
  if (lane != 0) return;
  const float s = h.scale[i];
  float r = 1.f / (sqrtf(fmaxf(lam, 0.f)) + h.eps * s);
  if (!isfinite(lam) || !isfinite(r)) {
    r = 1.f;
    if (h.status) atomicOr(h.status, SMUON_DEV_NONFINITE_NORM);
  }
  h.rscale[i] = r;
}

}  // namespace smuon
