// kernels.cuh -- declarations shared by the host ABI and the kernel files.
#pragma once

#include "plan.cuh"

namespace smuon {

// ---- plan upload: the plan bytes travel in kernel parameters
constexpr int kUploadBytes = 16384;
struct alignas(16) UploadChunk {
  void* dst;
  int32_t bytes;  // multiple of 16
  int32_t pad[1];
  alignas(16) unsigned char data[kUploadBytes];
};

// ---- elementwise tables (sign / vote / update / Lion), carried in kernel parameters
constexpr int kEwMaxLayers = 64;
constexpr int kEwMaxSrcs = 256;  // keeps the parameter block near 10 KB (launch cost grows with it)

struct EwSrc {
  const void* ptr;
  int64_t ld;
};

struct EwLayer {
  void* w;                 // weights (in/out), or unused
  int64_t w_ld;
  int64_t n;               // entries = rows * cols
  int64_t chunk_begin;     // first 8-entry chunk of this layer in the launch
  uint32_t* packed_out;    // nullable [M][words]
  int64_t words;           // packed words per worker
  int8_t* vote_out;        // nullable [n]
  void* aux;               // Lion mean output (f32, contiguous)
  int32_t w_dtype;
  int32_t vec;             // all operands contiguous and 16-byte aligned
  int32_t vec_aux;
  int32_t src_first;       // first entry of this layer in srcs[]
  int32_t rows, cols;
  uint32_t key0, key1;     // counter-based gradient stream keys (harness draws; key1 also for LionMuon)
};

struct EwTable {
  int32_t n_layers, M, tie, src_dtype;
  int32_t any_packed;
  int32_t test_starve;     // failure-detection test: the bulk-copy vote's producer issues nothing, short waits
  int32_t* status;         // nullable: SMUON_DEV_* bits (the bulk-copy vote's bounded waits)
  float eta, beta1, beta2, c1, c2;
  int32_t gen_on;          // LionMuon: gradients drawn in-kernel instead of read (srcs hold no G)
  uint32_t gen_seed;       // key word 0 of worker k = gen_seed + k
  uint32_t gen_step;       // counter word 2
  float gen_sigma;
  int32_t ghat_out;        // LionMuon vote-based Muon step: write each worker's G_hat (aux + k * n), no mean
  int64_t total_chunks;
  EwLayer layers[kEwMaxLayers];
  EwSrc srcs[kEwMaxSrcs];
};

__device__ __forceinline__ uint32_t pack_bf16x2_rn(float lo, float hi) {
  __nv_bfloat162 t = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&t);
}

// ---- kernels
__global__ void k_plan_upload(const __grid_constant__ UploadChunk c);
__global__ void k_momentum(const Plan* plan, const int32_t* skip);  // 256 threads per CTA
constexpr int kMomSlots = 8;  // sum-of-squares partials per 64x64 momentum tile (one per warp of k_momentum)
__global__ void k_norm_finalize(const Plan* plan, const int32_t* skip);
cudaError_t launch_vote_update(const EwTable& tb, bool popcount, int grid, int sms, cudaStream_t s);
bool bits_tma_eligible(const EwTable& tb);  // the 1-bit vote of this launch takes its bulk-copy form
__global__ void k_sign_pack(const __grid_constant__ EwTable tb, uint32_t* packed, int8_t* signs);
__global__ void k_vote(const uint32_t* packed, const int8_t* signs, int M, int64_t N, int64_t words,
                       int tie, int8_t* vote);
__global__ void k_update_src(const __grid_constant__ EwTable tb);
__global__ void k_harness_gaussian(const __grid_constant__ EwTable tb);

// spectral scaling (k_spectral.cu)
constexpr int kLanczosSteps = 64;  // at most; a matrix stops once its largest Ritz value has converged
__host__ __device__ constexpr int64_t lz_stride(int m) { return (m + 3) & ~3; }  // floats per Lanczos vector
__global__ void k_lz_start(const Plan* plan, const int32_t* skip);
__global__ void k_lz_matvec(const Plan* plan, int j, const int32_t* skip);
__global__ void k_lz_step(const Plan* plan, int j, const int32_t* skip);
__global__ void k_lz_finish(const Plan* plan, const int32_t* skip);
__global__ void k_lz_compact(const Plan* plan, int j, const int32_t* skip);
__global__ void k_lion_sign(const __grid_constant__ EwTable tb);
__global__ void k_lion_mean(const __grid_constant__ EwTable tb);
__global__ void k_probe_finalize(const Plan* plan);
__global__ void k_probe_nocache(float* d_err, int32_t* d_accept, cachemuon_counters* counters);

// GEMM stage kernels (grouped, persistent)
__global__ void k_gemm_simt_f32(const Plan* plan, int stage, int iter, const int32_t* skip);
__global__ void k_gemm_simt_bf16(const Plan* plan, int stage, int iter, const int32_t* skip);

// tcgen05 kernel entry (host-side launcher lives in k_gemm_tc.cu)
cudaError_t launch_gemm_tc(const Plan* d_plan, const PlanHeader& h, int stage, int iter,
                           const int32_t* skip, int num_sms, cudaStream_t s);
constexpr int kProbeSlots = 16;  // residual partial sums per probe tile (one per epilogue warp of either SM of a pair)
constexpr int kTcBM = 128;
// tile width of the split-BF16 stages: 128 x 256 tiles with two 96 KB ring stages (hi and lo parts of both
// operands) beat 128 x 128 tiles with three of 64 KB (4096^2, five quintic steps: 3.69 against 4.24 ms)
constexpr int kSplitBN = 256;
int tc_tile_n(int stage, uint32_t flags);  // 128 (symmetric stages, split mode) or 256
int tc_pair_clusters();                    // clusters of the SM-pair GEMM kernel the device holds at once
// a plan runs its tensor-core stages on SM pairs when every matrix's smaller side is at least this
constexpr int kPairMinM = 256;
constexpr int kSimtBM = 64;
constexpr int kSimtBN = 64;

}  // namespace smuon
