// k_spectral.cu -- spectral-norm normalisation of the Newton-Schulz input.
//
// The "SignMuon" summary (section 4) allows the spectral norm in place of the
// Frobenius norm. The first Gram stage already holds A_0 = s^2 X X^T (s the
// Frobenius scale), whose largest eigenvalue is (s ||M||_2)^2. A Lanczos
// iteration with full reorthogonalisation estimates it for every matrix of
// the batch at once; the first step's epilogues then rescale by
// r = 1 / (sqrt(lambda_max) + eps s), so that X_0 = s r M = M / (||M||_2 + eps).
//
// Per Lanczos step j: w = A v_j (k_lz_matvec: one warp per row, all matrices),
// then alpha_j = w.v_j, w -= alpha_j v_j + beta_{j-1} v_{j-1}, w is
// orthogonalised against every earlier v, beta_j = ||w||, v_{j+1} = w / beta_j
// (k_lz_step: one CTA per matrix). The largest eigenvalue of the tridiagonal
// (alpha, beta) matrix is found by bisection on its Sturm counts (k_lz_finish).
#include "kernels.cuh"

namespace smuon {

namespace {

__device__ __forceinline__ float* lz_vec(const PlanHeader& h, const MatDesc& md, int j) {
  const GroupDesc& g = h.groups[md.group];
  return h.lz + md.lz_off + (int64_t)j * g.m;
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

// matrix of a flattened Lanczos row (binary search over the compact row prefix)
__device__ __forceinline__ int lz_mat_of_row(const PlanHeader& h, int64_t row) {
  int lo = 0, hi = h.n_mats - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (h.lz_rows[mid] <= row) lo = mid; else hi = mid - 1;
  }
  return lo;
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

// w = A v_j for every matrix: one warp per row of A (f32, in its group's buffer)
__global__ void __launch_bounds__(256) k_lz_matvec(const Plan* plan, int j, const int32_t* skip) {
  if (skip && *skip) return;
  const PlanHeader& h = plan->h;
  const int lane = threadIdx.x & 31;
  const int64_t warps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const int64_t total = h.lz_rows[h.n_mats];
  for (int64_t row = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; row < total; row += warps) {
    const int i = lz_mat_of_row(h, row);
    const MatDesc& md = h.mats[i];
    const GroupDesc& g = h.groups[md.group];
    const int r = (int)(row - h.lz_rows[i]);
    const float* a = g.af + ((int64_t)md.z * g.m + r) * g.ldm;
    const float* v = lz_vec(h, md, j);
    float acc = 0.f;
    for (int k = lane; k < g.m; k += 32) acc += a[k] * v[k];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) lz_vec(h, md, kLanczosSteps + 1)[r] = acc;  // the work vector w
  }
}

// one Lanczos step per matrix (one CTA each)
__global__ void __launch_bounds__(256) k_lz_step(const Plan* plan, int j, const int32_t* skip) {
  if (skip && *skip) return;
  const PlanHeader& h = plan->h;
  __shared__ float red[8];
  for (int i = blockIdx.x; i < h.n_mats; i += gridDim.x) {
    const MatDesc& md = h.mats[i];
    const int m = h.groups[md.group].m;
    float* ab = h.lz_ab + (int64_t)i * 2 * kLanczosSteps;  // alpha[0..K), beta[K..2K)
    float* w = lz_vec(h, md, kLanczosSteps + 1);
    const float* vj = lz_vec(h, md, j);
    if (j > 0 && ab[kLanczosSteps + j - 1] == 0.f) {  // an earlier step broke down: nothing to add
      if (threadIdx.x == 0) { ab[j] = 0.f; ab[kLanczosSteps + j] = 0.f; }
      continue;
    }
    float p = 0.f;
    for (int k = threadIdx.x; k < m; k += blockDim.x) p += w[k] * vj[k];
    const float alpha = block_sum(p, red);
    const float bprev = j > 0 ? ab[kLanczosSteps + j - 1] : 0.f;
    const float* vp = j > 0 ? lz_vec(h, md, j - 1) : vj;
    for (int k = threadIdx.x; k < m; k += blockDim.x) w[k] -= alpha * vj[k] + bprev * vp[k];
    __syncthreads();
    // full reorthogonalisation against v_0 .. v_j
    for (int t = 0; t <= j; ++t) {
      const float* vt = lz_vec(h, md, t);
      float q = 0.f;
      for (int k = threadIdx.x; k < m; k += blockDim.x) q += w[k] * vt[k];
      const float c = block_sum(q, red);
      for (int k = threadIdx.x; k < m; k += blockDim.x) w[k] -= c * vt[k];
      __syncthreads();
    }
    float ss = 0.f;
    for (int k = threadIdx.x; k < m; k += blockDim.x) ss += w[k] * w[k];
    const float beta = sqrtf(block_sum(ss, red));
    const bool ok = beta > 1e-6f * fabsf(alpha) && beta > 1e-30f && j + 1 < kLanczosSteps;
    if (ok) {
      float* vn = lz_vec(h, md, j + 1);
      const float inv = 1.f / beta;
      for (int k = threadIdx.x; k < m; k += blockDim.x) vn[k] = w[k] * inv;
    }
    if (threadIdx.x == 0) { ab[j] = alpha; ab[kLanczosSteps + j] = ok ? beta : 0.f; }
    __syncthreads();
  }
}

// Sturm count: eigenvalues of the k x k tridiagonal matrix below x
__device__ __forceinline__ int sturm_below(const float* alpha, const float* beta, int k, double x) {
  int count = 0;
  double d = 1.0;
  for (int i = 0; i < k; ++i) {
    const double b2 = i > 0 ? (double)beta[i - 1] * beta[i - 1] : 0.0;
    d = ((double)alpha[i] - x) - (i > 0 ? b2 / d : 0.0);
    if (d == 0.0) d = -1e-300;
    if (d < 0.0) ++count;
  }
  return count;
}

// lambda_max of each matrix's tridiagonal matrix by bisection, then r = 1 / (sqrt(lambda) + eps s)
__global__ void k_lz_finish(const Plan* plan, const int32_t* skip) {
  if (skip && *skip) return;
  const PlanHeader& h = plan->h;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < h.n_mats; i += gridDim.x * blockDim.x) {
    const float* alpha = h.lz_ab + (int64_t)i * 2 * kLanczosSteps;
    const float* beta = alpha + kLanczosSteps;
    int k = 1;  // the Krylov dimension actually built: steps up to the first breakdown
    while (k < kLanczosSteps && beta[k - 1] != 0.f) ++k;
    double lo = 0.0, hi = 0.0;
    for (int t = 0; t < k; ++t) {
      const double rad = (t > 0 ? fabs((double)beta[t - 1]) : 0.0) + (t + 1 < k ? fabs((double)beta[t]) : 0.0);
      hi = fmax(hi, (double)alpha[t] + rad);
      lo = fmin(lo, (double)alpha[t] - rad);
    }
    for (int it = 0; it < 100 && hi - lo > 1e-12 * fmax(1.0, fabs(hi)); ++it) {
      const double mid = 0.5 * (lo + hi);
      if (sturm_below(alpha, beta, k, mid) == k) hi = mid; else lo = mid;
    }
    const float lam = (float)hi;  // 0 for a zero matrix: then s r = 1/eps, as in the Frobenius case
    const float s = h.scale[i];
    float r = 1.f / (sqrtf(fmaxf(lam, 0.f)) + h.eps * s);
    if (!isfinite(lam) || !isfinite(r)) {
      r = 1.f;
      if (h.status) atomicOr(h.status, SMUON_DEV_NONFINITE_NORM);
    }
    h.rscale[i] = r;
  }
}

}  // namespace smuon
