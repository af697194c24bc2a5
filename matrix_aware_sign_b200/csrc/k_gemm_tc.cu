// k_gemm_tc.cu -- grouped Newton-Schulz GEMM stages on the sm_100a tensor cores.
//
// One persistent kernel per stage (all layers x workers in one launch); each
// CTA walks its own list of tiles from the plan's schedule. Per CTA (320
// threads, one per SM):
//   warp 0      TMA producer: 128B-swizzled tiles of A (K-major) and B
//               (K-major, or MN-major for the X / Q right operand) into a
//               shared-memory ring (full/empty mbarriers): 4 stages of
//               128 x 64 + 256 x 64 bf16 in plain mode, 2 stages of hi and
//               lo parts of 128 x 64 + 256 x 64 in split mode
//   warp 1      TMEM allocation and the single MMA-issuing thread:
//               tcgen05.mma.cta_group::1.kind::f16, BF16 x BF16 -> FP32,
//               M = 128, N = BN = 256, K = 16 per
//               instruction (three per step in split mode: hi*hi, hi*lo,
//               lo*hi), into one of two TMEM accumulators of BN columns
//   warps 2-9   epilogue, two warps per TMEM lane group (one per half of the
//               columns): tcgen05.ld 32 lanes x 32 columns at a time, stage
//               algebra in FP32 (epilogue.cuh), global stores
// The two accumulators let the epilogue of tile i overlap the MMAs of tile
// i+1. Every mbarrier wait is bounded; on expiry the CTA records
// SMUON_DEV_WAIT_TIMEOUT, drains its own copies and MMAs, frees TMEM and exits.
//
// SM pairs (k_gemm_tc2, clusters of two CTAs): one 256 x 256 tile per pair,
// tcgen05.mma.cta_group::2 with M = 256 issued by the even CTA. Each CTA
// stages its own 128 rows of A and its own 128-row half of the B tile (by
// TMA, the copies of both CTAs completing on the even CTA's full barrier) and
// holds its 128 x 256 half of the accumulator in its own TMEM; the MMA
// commits arrive on both CTAs' barriers, and both CTAs' epilogue warps
// release an accumulator at the even CTA. Per SM this halves the shared-
// memory operand traffic of a 256-wide tile (each SM reads A once and half of
// B), the limit of the single-SM 128 x 256 form.
#include "epilogue.cuh"

namespace smuon {
namespace tc {

constexpr int BM = kTcBM;
constexpr int THREADS = 320;  // TMA warp, MMA warp, 8 epilogue warps (+ one source warp for B X)
constexpr int SRC_SLOTS = 2;                // B X epilogue source ring
constexpr int SRC_BYTES = BM * 32 * 4;      // one 128 x 32 f32 chunk of X (or its transpose)

// plain BF16: one hi tile per operand; split BF16: hi and lo tiles per operand
// (x = x_hi + x_lo, product ~ A_hi B_hi + A_hi B_lo + A_lo B_hi).
// Tiles are 128 x 256 (kBN = 256; the symmetric stages use them over the
// triangle, the others a full grid). The ring takes 192 KB of shared memory,
// or about 144 KB (kShallow, plain mode) for stages whose K is short: a tile
// then needs few k-blocks in flight, and the shared memory left to the L1
// cache serves the epilogue's row-per-lane global accesses. Split mode keeps
// the 192 KB ring (two stages of 96 KB).
// k-blocks are 64 deep: K-major rows of 64 bf16 (128 bytes) with the 128-byte swizzle
template <bool kSplit, int kBN, bool kShallow, bool kSrc, bool kPair = false>
struct Cfg {
  static constexpr int PARTS = kSplit ? 2 : 1;
  static constexpr int BN = kBN;
  static constexpr int BK = 64;
  static constexpr int B_ROWS = kPair ? kBN / 2 : kBN;  // rows of the B tile this CTA stages
  static constexpr int A_BYTES = BM * BK * 2;   // one bf16 tile of A (128 rows x BK)
  static constexpr int B_BYTES = B_ROWS * BK * 2;
  static constexpr int MN_BOX = 64 * BK * 2;     // one {64, BK} box of an MN-major B operand
  static constexpr int STAGE_BYTES = PARTS * (A_BYTES + B_BYTES);
  static constexpr int STAGES = ((kShallow ? 144 : 192) * 1024) / STAGE_BYTES;
  static constexpr int TMEM_COLS = 2 * kBN;
  static constexpr int NTHREADS = THREADS + (kSrc ? 32 : 0);
  static constexpr int SRC_RING = kSrc ? SRC_SLOTS * SRC_BYTES : 0;
  // the generic epilogue's transpose buffers (symmetric stages): 32 x 33 floats per epilogue warp
  static constexpr int XPOSE = kSrc ? 0 : 8 * 32 * 33 * 4;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + SRC_RING + 1024 /*align*/ + 256 /*barriers*/ + XPOSE;
};
constexpr unsigned long long kWaitCycles = 1ull << 32;  // ~2 s at 2 GHz: the exit drains' budget
template <int V>
struct StageTag {
  static constexpr int value = V;
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
  return ok != 0;
}

// bounded wait: false when the budget (SM clocks) ran out or another role aborted
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          unsigned long long budget) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = clock64();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 63) == 0) {
      if (*abort_flag) return false;
      if (clock64() - t0 > budget) return false;
    }
  }
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, int c0, int c1, int c2,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];"
      ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(bar)
      : "memory");
}

// SM-pair form: the copy lands in this CTA's shared memory and completes on the mbarrier at cluster
// address bar_cluster (the even CTA's full barrier)
__device__ __forceinline__ void tma_load_3d_pair(uint32_t dst, const CUtensorMap* map, int c0, int c1, int c2,
                                                 uint32_t bar_cluster) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];"
      ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(bar_cluster)
      : "memory");
}

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// cluster address of the same shared-memory location in the even CTA of the pair
__device__ __forceinline__ uint32_t at_rank0(uint32_t saddr) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, 0;" : "=r"(r) : "r"(saddr));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Relaxed arrives for the epilogue's releases of a source slot or an accumulator: what must precede them
// is the warp's reads of that shared memory (whose values the warp has already used) or of that tensor
// memory (completed by tcgen05.wait::ld and ordered by tcgen05.fence::before_thread_sync). A release arrive
// would also wait for every global store the warp has issued, which the consumers of these barriers (the
// source producer and the MMA issuer) never read.
__device__ __forceinline__ void mbar_arrive_relaxed(uint32_t bar) {
  asm volatile("mbarrier.arrive.relaxed.cta.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t bar_cluster) {
  asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster) : "memory");
}

__device__ __forceinline__ void tensormap_acquire(const CUtensorMap* map) {
  asm volatile("fence.proxy.tensormap::generic.acquire.gpu [%0], 128;" ::"l"(reinterpret_cast<uint64_t>(map))
               : "memory");
}

// shared-memory matrix descriptors (tcgen05 format: version 1, 128B swizzle)
__device__ __forceinline__ uint64_t desc_sw128(uint32_t saddr, uint32_t lbo_bytes) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFF);
  d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFF) << 16;
  d |= (uint64_t)(1024 >> 4) << 32;  // 8-row group stride
  d |= (uint64_t)1 << 46;            // descriptor version for sm_100
  d |= (uint64_t)2 << 61;            // SWIZZLE_128B
  return d;
}
// K-major descriptor of a 64-deep tile at k-step kk (16 elements = 32 bytes into each 128-byte row)
__device__ __forceinline__ uint64_t desc_k(uint32_t saddr, int kk) { return desc_sw128(saddr + kk * 32, 16); }

// instruction descriptor: BF16 x BF16 -> F32, A K-major, B K- or MN-major, m x n (m = 128, or 256 for a
// pair of SMs)
__host__ __device__ constexpr uint32_t make_idesc(uint32_t b_mn, int n, int m = BM) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (b_mn << 16) | ((uint32_t)(n >> 3) << 17) |
         ((uint32_t)(m >> 4) << 24);
}

__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                         uint32_t accum) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n"
      ::"r"(d_tmem), "l"(a), "l"(b), "r"(idesc), "r"(accum));
}
__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}
// SM pairs: the 256-row MMA (A rows and B columns from both CTAs, D in both TMEMs), and its commit,
// which arrives on the barrier at the same offset in both CTAs
__device__ __forceinline__ void mma_bf16_pair(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                              uint32_t accum) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n}\n"
      ::"r"(d_tmem), "l"(a), "l"(b), "r"(idesc), "r"(accum));
}
__device__ __forceinline__ void mma_commit_pair(uint32_t bar) {
  const uint16_t both = 3;
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;"
      ::"r"(bar), "h"(both) : "memory");
}
template <bool kPair>
__device__ __forceinline__ void mma_issue(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t accum) {
  if constexpr (kPair) mma_bf16_pair(d, a, b, idesc, accum);
  else mma_bf16(d, a, b, idesc, accum);
}
template <bool kPair>
__device__ __forceinline__ void commit_to(uint32_t bar) {
  if constexpr (kPair) mma_commit_pair(bar);
  else mma_commit(bar);
}
__device__ __forceinline__ void fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
        "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
        "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float* v) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// Split form of a 32-lane x 16-column accumulator load: issue now, wait later. The wait names the
// destination registers as operands, so no use of them can be scheduled above it.
__device__ __forceinline__ void tmem_ld16_issue(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait(uint32_t (&r)[16]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                 "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                 "+r"(r[15])
               :
               : "memory");
}

// operands of one tile: tensor maps, coordinates, K extent
struct TcOps {
  const CUtensorMap* ma;
  const CUtensorMap* mb;
  int za, zb;
  int zlo;   // split mode: the lo part of matrix z is matrix z + zlo of the same map
  int K;
  int b_mn;
};

// brows: rows of the B tile one CTA stages (256 for a single-SM 128 x 256 tile, 128 for each CTA of a pair)
__device__ __forceinline__ TcOps tc_ops(const PlanHeader& h, const TileCtx& t, int iter, int brows) {
  const GroupDesc& g = *t.g;
  TcOps o;
  o.za = o.zb = t.z;
  o.zlo = g.count;
  const bool wide = brows == 256;  // K-major B tiles of 256 rows use the {64, 256} boxes
  switch (t.stage) {
    case ST_GRAM:
      o.ma = &h.tmaps[g.tm_x_k[iter & 1]];
      o.mb = &h.tmaps[wide ? g.tm_x_kw[iter & 1] : g.tm_x_k[iter & 1]];
      o.K = g.n; o.b_mn = 0; break;
    case ST_POLY:
      o.ma = &h.tmaps[g.tm_a_k];
      o.mb = &h.tmaps[wide ? g.tm_a_kw : g.tm_a_k];
      o.K = g.m; o.b_mn = 0; break;
    case ST_AXPY: o.ma = &h.tmaps[g.tm_b_k]; o.mb = &h.tmaps[g.tm_x_mn[iter & 1]]; o.K = g.m; o.b_mn = 1; break;
    case ST_QAXPY: o.ma = &h.tmaps[g.tm_b_k]; o.mb = &h.tmaps[g.tm_q_mn[iter & 1]]; o.K = g.m; o.b_mn = 1; break;
    case ST_REUSE: o.ma = &h.tmaps[g.tm_uq_k]; o.za = 0; o.mb = &h.tmaps[g.tm_x_mn[0]]; o.K = g.m; o.b_mn = 1; break;
    case ST_AA1:  // B * A with A symmetric: its rows are the K-major right operand
      o.ma = &h.tmaps[g.tm_b_k];
      o.mb = &h.tmaps[wide ? g.tm_a_kw : g.tm_a_k];
      o.K = g.m; o.b_mn = 0; break;
    case ST_QX:  // Q_K (K-major rows, hi and lo parts) times X_0 (MN-major)
      o.ma = &h.tmaps[g.tm_q_k[iter & 1]];
      o.mb = &h.tmaps[g.tm_x_mn[0]];
      o.K = g.m; o.b_mn = 1; break;
    case ST_AA2:  // B * T, T symmetric
      o.ma = &h.tmaps[g.tm_b_k];
      o.mb = &h.tmaps[wide ? g.tm_t_kw : g.tm_t_k];
      o.K = g.m; o.b_mn = 0; break;
    default:  // ST_PROBE
      o.ma = &h.tmaps[g.tm_x_k[1]];
      o.mb = &h.tmaps[wide ? g.tm_x_kw[1] : g.tm_x_k[1]];
      o.K = g.n; o.b_mn = 0; break;
  }
  return o;
}

template <bool kSplit, int kBN, bool kShallow, bool kSrc, bool kPair>
__device__ __forceinline__ void gemm_tc_body(const Plan* plan, int stage, int iter) {
  using C = Cfg<kSplit, kBN, kShallow, kSrc, kPair>;
  constexpr int STAGES = C::STAGES;
  constexpr int STAGE_BYTES = C::STAGE_BYTES;
  constexpr int PARTS = C::PARTS;
  constexpr int B_BYTES = C::B_BYTES;
  constexpr int A_BYTES = C::A_BYTES;
  constexpr int BK = C::BK;
  constexpr int B_ROWS = C::B_ROWS;
  const PlanHeader& h = plan->h;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  unsigned char* base_ptr = smem_raw + (base - raw);
  const uint32_t src_base = base + STAGES * STAGE_BYTES;  // B X source ring (kSrc), 1024-aligned
  const uint32_t bar0 = src_base + C::SRC_RING;
  // barrier layout (8 bytes each): full[S], empty[S], tfull[2], tempty[2], done, sfull[2], sempty[2]
  const uint32_t full_bar = bar0, empty_bar = bar0 + 8 * STAGES;
  const uint32_t tfull_bar = bar0 + 16 * STAGES, tempty_bar = tfull_bar + 16, done_bar = tempty_bar + 16;
  const uint32_t sfull_bar = done_bar + 8, sempty_bar = sfull_bar + 8 * SRC_SLOTS;
  unsigned char* misc = base_ptr + STAGES * STAGE_BYTES + C::SRC_RING + 8 * (2 * STAGES + 5 + 2 * SRC_SLOTS);
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 4);
  float* xpose = reinterpret_cast<float*>(base_ptr + STAGES * STAGE_BYTES + C::SRC_RING + 256);  // after the barriers
  static_assert(8 * (2 * STAGES + 5 + 2 * SRC_SLOTS) + 8 <= 256, "barriers and flags fit their 256 bytes");
  static_assert(C::SMEM_BYTES <= 232448, "shared memory per CTA");

  // SM pairs: rank 0 issues the MMAs and owns the full and tempty barriers that count both CTAs
  const uint32_t rank = kPair ? cluster_rank() : 0u;
  const bool leader = rank == 0;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) { mbar_init(full_bar + 8 * s, 1); mbar_init(empty_bar + 8 * s, 1); }
    // tempty: every epilogue thread arrives (single SM), or one arrive per epilogue warp of both CTAs
    for (int a = 0; a < 2; ++a) { mbar_init(tfull_bar + 8 * a, 1); mbar_init(tempty_bar + 8 * a, kPair ? 16 : 256); }
    mbar_init(done_bar, 1);
    for (int q = 0; q < SRC_SLOTS; ++q) { mbar_init(sfull_bar + 8 * q, 1); mbar_init(sempty_bar + 8 * q, 8); }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    if constexpr (kPair) {
      asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32((const void*)tmem_slot)),
                   "r"(C::TMEM_COLS));
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
    } else {
      asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32((const void*)tmem_slot)),
                   "r"(C::TMEM_COLS));
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
  }
  fence_before();
  if constexpr (kPair) {
    __syncwarp();
    cluster_sync_all();  // both CTAs' barriers exist before either signals the other's
  } else {
    __syncthreads();
  }
  fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // split mode: both parts of every operand, except in the plain leading steps (hi parts only); the
  // producer and the MMA issuer take the same decision, per tile, from the tile's group
  const unsigned long long budget = h.wait_cycles;
  // this CTA's tiles (host-balanced list; every role walks the same one; both CTAs of a pair walk the
  // pair's list, whose tiles are 256 rows high: this CTA takes rows 128 * (2 tm + rank) ...)
  const int list = kPair ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
  const int32_t* tiles = h.sched + h.sched_off[stage];
  const int t_begin = h.sched_begin[h.sched_boff[stage] + list];
  const int t_end = h.sched_begin[h.sched_boff[stage] + list + 1];
  // tile i of the list: its tile coordinates, its first column and its width (kBN, or kBN / 2 for a half tile
  // of a B X stage's last wave)
  auto tile_at = [&](int i, int& tm, int& tn, int& cbase, int& bw) {
    const int32_t e = tiles[i];
    const bool halfw = (e & kHalfTileFlag) != 0;
    const TileCtx t = make_ctx(h, stage, iter, e & (kHalfTileSide - 1), tm, tn);
    if (kPair) tm = 2 * tm + (int)rank;
    bw = halfw ? kBN / 2 : kBN;
    cbase = tn * kBN + ((halfw && (e & kHalfTileSide)) ? kBN / 2 : 0);
    return t;
  };

  if (warp == 0) {
    // ---------------- TMA producer (lane 0)
    int s = 0;
    uint32_t ph = 0;
    uint32_t armed = 0, last_par = 0;  // per-stage bit sets for the exit drain
    bool ok = true;
    for (int i = t_begin; i < t_end && ok && !h.starve_tc; ++i) {
      int tm, tn, cbase, bw;
      const TileCtx t = tile_at(i, tm, tn, cbase, bw);
      const int parts = (kSplit && !plain_lead_stage(h.flags, stage, iter, t.g->m)) ? PARTS : 1;
      if (lane == 0) {
        const TcOps o = tc_ops(h, t, iter, B_ROWS);
        tensormap_acquire(o.ma);
        tensormap_acquire(o.mb);
        const int nk = (o.K + BK - 1) / BK;
        const int brows = kPair ? bw / 2 : bw;           // B columns (MN-major) this CTA stages for the tile
        const int brow = cbase + (int)rank * brows;      // first B row (K-major) or column (MN-major) staged here
        const int b_bytes = brows * BK * 2;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(empty_bar + 8 * s, ph ^ 1u, abort_flag, budget)) { ok = false; break; }
          const uint32_t fb = full_bar + 8 * s;
          const uint32_t fb_tx = kPair ? at_rank0(fb) : fb;
          if (leader) {  // the pair's full barrier expects both CTAs' bytes
            mbar_expect_tx(fb, (kPair ? 2 : 1) * parts * (A_BYTES + b_bytes));
            armed |= 1u << s;
            last_par = (last_par & ~(1u << s)) | (ph << s);
          }
          const uint32_t sa = base + s * STAGE_BYTES, sb = sa + PARTS * A_BYTES;
          for (int part = 0; part < parts; ++part) {
            const int za = o.za + part * o.zlo, zb = o.zb + part * o.zlo;
            const uint32_t da = sa + part * A_BYTES, db = sb + part * B_BYTES;
            if constexpr (kPair) {
              tma_load_3d_pair(da, o.ma, kb * BK, tm * BM, za, fb_tx);
              if (o.b_mn) {
#pragma unroll
                for (int q = 0; q < B_ROWS / 64; ++q)
                  if (q < brows / 64) tma_load_3d_pair(db + q * C::MN_BOX, o.mb, brow + 64 * q, kb * BK, zb, fb_tx);
              } else {
                tma_load_3d_pair(db, o.mb, kb * BK, brow, zb, fb_tx);
              }
            } else {
              tma_load_3d(da, o.ma, kb * BK, tm * BM, za, fb);
              if (o.b_mn) {
#pragma unroll
                for (int q = 0; q < B_ROWS / 64; ++q)
                  if (q < brows / 64) tma_load_3d(db + q * C::MN_BOX, o.mb, brow + 64 * q, kb * BK, zb, fb);
              } else {
                tma_load_3d(db, o.mb, kb * BK, brow, zb, fb);
              }
            }
          }
          if (++s == STAGES) { s = 0; ph ^= 1u; }
        }
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    }
    if (lane == 0) {
      if (!ok) {
        *abort_flag = 1;
        if (h.status) atomicOr(h.status, SMUON_DEV_WAIT_TIMEOUT);
      }
      // drain: every armed stage's last phase must have landed before exit (with SM pairs the even
      // CTA's barriers count the copies of both CTAs, and the final cluster barrier holds the odd CTA)
      for (int q = 0; q < STAGES; ++q)
        if (armed & (1u << q)) {
          const uint32_t p = (last_par >> q) & 1u;
          const unsigned long long t0 = clock64();
          while (!mbar_try_wait(full_bar + 8 * q, p) && clock64() - t0 < kWaitCycles) {}
        }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ---------------- MMA issuer
      int s = 0;
      uint32_t ph = 0;
      int acc = 0;
      uint32_t acc_ph = 0;
      bool ok = true;
      for (int i = t_begin; i < t_end && ok; ++i) {
        int tm, tn, cbase, bw;
        const TileCtx t = tile_at(i, tm, tn, cbase, bw);
        const TcOps o = tc_ops(h, t, iter, B_ROWS);
        const uint32_t idesc = make_idesc((uint32_t)o.b_mn, bw, kPair ? 2 * BM : BM);
        const bool use_lo = kSplit && !plain_lead_stage(h.flags, stage, iter, t.g->m);
        if (!mbar_wait(tempty_bar + 8 * acc, acc_ph ^ 1u, abort_flag, budget)) { ok = false; break; }
        fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * kBN);
        const int nk = (o.K + BK - 1) / BK;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(full_bar + 8 * s, ph, abort_flag, budget)) { ok = false; break; }
          fence_after();
          const uint32_t sa = base + s * STAGE_BYTES, sb = sa + PARTS * A_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t ad = desc_k(sa, kk);
            const uint64_t bd = o.b_mn ? desc_sw128(sb + kk * 2048, C::MN_BOX) : desc_k(sb, kk);
            mma_issue<kPair>(d_tmem, ad, bd, idesc, (kb | kk) != 0);
            if (kSplit && use_lo) {
              const uint64_t adl = desc_k(sa + A_BYTES, kk);
              const uint32_t sbl = sb + B_BYTES;
              const uint64_t bdl = o.b_mn ? desc_sw128(sbl + kk * 2048, C::MN_BOX) : desc_k(sbl, kk);
              mma_issue<kPair>(d_tmem, ad, bdl, idesc, 1u);   // A_hi * B_lo
              mma_issue<kPair>(d_tmem, adl, bd, idesc, 1u);   // A_lo * B_hi
            }
          }
          commit_to<kPair>(empty_bar + 8 * s);  // frees the smem slot (of both CTAs) once these MMAs have read it
          if (++s == STAGES) { s = 0; ph ^= 1u; }
        }
        if (!ok) break;
        commit_to<kPair>(tfull_bar + 8 * acc);  // accumulator ready for the epilogue(s)
        if (++acc == 2) { acc = 0; acc_ph ^= 1u; }
      }
      if (!ok) {
        *abort_flag = 1;
        if (h.status) atomicOr(h.status, SMUON_DEV_WAIT_TIMEOUT);
      }
      // all MMAs issued by this thread complete before TMEM is released
      commit_to<kPair>(done_bar);
      const unsigned long long t0 = clock64();
      while (!mbar_try_wait(done_bar, 0) && clock64() - t0 < kWaitCycles) {}
    } else if (kPair && lane == 0) {
      // odd CTA of a pair: the even CTA's last commit also arrives here once its MMAs (which write this
      // CTA's TMEM) are complete
      const unsigned long long t0 = clock64();
      while (!mbar_try_wait(done_bar, 0) && clock64() - t0 < kWaitCycles) {}
    }
  } else if (kSrc && warp == 10) {
    if (lane == 0) {
      // ---------------- B X source producer: the tile's X (f32, 128 rows x 32 columns per chunk, in
      // chunk order) into a two-slot ring that all eight epilogue warps drain together
      int k = 0;
      uint32_t armed = 0, last_par = 0;
      bool ok = true;
      const bool hilo = (h.flags & SMUON_NS_SPLIT_BF16) != 0;
      for (int i = t_begin; i < t_end && ok && !h.starve_tc; ++i) {
        int tm, tn, cbase, bw;
        const TileCtx t = tile_at(i, tm, tn, cbase, bw);
        const bool first = iter == 0;
        const CUtensorMap* map = first ? &h.tmaps[t.md->tm_src] : &h.tmaps[t.g->tm_xf[iter & 1]];
        const bool tall = first && t.md->tall;
        tensormap_acquire(map);
        for (int c = 0; c < bw / 32; ++c, ++k) {
          const int slot = k & 1;
          const uint32_t ph = (uint32_t)(k >> 1) & 1u;
          if (!mbar_wait(sempty_bar + 8 * slot, ph ^ 1u, abort_flag, budget)) { ok = false; break; }
          const uint32_t fb = sfull_bar + 8 * slot;
          mbar_expect_tx(fb, SRC_BYTES);
          armed |= 1u << slot;
          last_par = (last_par & ~(1u << slot)) | (ph << slot);
          const uint32_t dst = src_base + slot * SRC_BYTES;
          const int col = cbase + c * 32;  // wide-form column of the chunk
          if (!first && hilo) {  // split mode: X as its bf16 hi part, then its lo part (matrix z + count)
            tma_load_3d(dst, map, col, tm * BM, t.z, fb);
            tma_load_3d(dst + SRC_BYTES / 2, map, col, tm * BM, t.z + t.g->count, fb);
          } else if (!first) {
            tma_load_3d(dst, map, col, tm * BM, t.z, fb);
          } else if (!tall) {
            tma_load_3d(dst, map, col, tm * BM, 0, fb);   // user rows = wide rows
          } else {
            tma_load_3d(dst, map, tm * BM, col, 0, fb);   // user rows = wide columns
          }
        }
      }
      if (!ok) {
        *abort_flag = 1;
        if (h.status) atomicOr(h.status, SMUON_DEV_WAIT_TIMEOUT);
      }
      for (int q = 0; q < SRC_SLOTS; ++q)
        if (armed & (1u << q)) {
          const uint32_t p = (last_par >> q) & 1u;
          const unsigned long long t0 = clock64();
          while (!mbar_try_wait(sfull_bar + 8 * q, p) && clock64() - t0 < kWaitCycles) {}
        }
    }
  } else if (warp >= 2 && warp < 10) {
    // ---------------- epilogue warps 2..9: two warps per TMEM lane group (one per half of the columns)
    const int ew = warp & 3;         // TMEM lane group this warp may access
    const int half = (warp - 2) >> 2;
    const int lrow = ew * 32 + lane;  // row within the tile
    int acc = 0;
    uint32_t acc_ph = 0;
    int kc = 0;
    bool ok = true;
    for (int i = t_begin; i < t_end && ok; ++i) {
      int tm, tn, cbase, bw;
      TileCtx t = tile_at(i, tm, tn, cbase, bw);
      if (!mbar_wait(tfull_bar + 8 * acc, acc_ph, abort_flag, budget)) { ok = false; break; }
      fence_after();
      float pacc = 0.f;
      if constexpr (kSrc) {
        // B X: every warp takes each 32-column chunk in turn (its lane group's 32 rows, one 16-column
        // half), with the X source from the shared-memory ring. The accumulator load of the next chunk
        // is in flight while this one is processed (two register sets, the loop unrolled by two).
        const float* ring = reinterpret_cast<const float*>(base_ptr + STAGES * STAGE_BYTES);
        const bool tall = iter == 0 && t.tall;
        const bool hilo = iter > 0 && t.split;  // the source is X's hi and lo parts, not an f32 master
        auto taddr = [&](int c) {
          return tmem_base + (uint32_t)(acc * kBN + c * 32 + 16 * half) + ((uint32_t)(ew * 32) << 16);
        };
        auto process = [&](int c, const uint32_t (&r)[16]) -> bool {
          const int slot = kc & 1;
          if (!mbar_wait(sfull_bar + 8 * slot, (uint32_t)(kc >> 1) & 1u, abort_flag, budget)) return false;
          float v[16], x[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) v[j] = __uint_as_float(r[j]);
          const float* sp = ring + slot * (SRC_BYTES / 4);
          if (hilo) {
            // split mode, steps >= 1: [128 rows][32 bf16] hi, then lo, with the 64-byte swizzle: 16-byte
            // unit u of row r sits at u ^ ((r >> 1) & 3); this lane's 16 columns are units 2 half, 2 half + 1
            const unsigned char* hp = reinterpret_cast<const unsigned char*>(sp) + lrow * 64;
            const unsigned char* lp = hp + SRC_BYTES / 2;
#pragma unroll
            for (int q = 0; q < 2; ++q) {
              const int u = ((2 * half + q) ^ ((lrow >> 1) & 3)) << 4;
              const uint4 wh = *reinterpret_cast<const uint4*>(hp + u);
              const uint4 wl = *reinterpret_cast<const uint4*>(lp + u);
              const uint32_t hw[4] = {wh.x, wh.y, wh.z, wh.w}, lw[4] = {wl.x, wl.y, wl.z, wl.w};
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                x[8 * q + 2 * j] = __uint_as_float(hw[j] << 16) + __uint_as_float(lw[j] << 16);
                x[8 * q + 2 * j + 1] = __uint_as_float(hw[j] & 0xffff0000u) + __uint_as_float(lw[j] & 0xffff0000u);
              }
            }
          } else if (!tall) {
            // [128 rows][32 f32] with the 128-byte swizzle: 16-byte unit u of row r sits at u ^ (r & 7)
            const unsigned char* rp = reinterpret_cast<const unsigned char*>(sp) + lrow * 128;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const float4 f = *reinterpret_cast<const float4*>(rp + (((4 * half + q) ^ (lrow & 7)) << 4));
              x[4 * q] = f.x; x[4 * q + 1] = f.y; x[4 * q + 2] = f.z; x[4 * q + 3] = f.w;
            }
          } else {
            // [32 user rows = wide columns][128 f32 = wide rows], no swizzle: lanes read along a row
#pragma unroll
            for (int j = 0; j < 16; ++j) x[j] = sp[(16 * half + j) * BM + lrow];
          }
          epi_axpy_src<16>(t, tm * BM + lrow, cbase + c * 32 + 16 * half, v, x);
          __syncwarp();
          if (lane == 0) mbar_arrive_relaxed(sempty_bar + 8 * slot);
          ++kc;
          return true;
        };
        static_assert((kBN / 32) % 2 == 0, "chunks are processed in pairs");
        uint32_t ra[16], rb[16];
        tmem_ld16_issue(taddr(0), ra);
        for (int c = 0; c < bw / 32 && ok; c += 2) {
          tmem_ld_wait(ra);
          tmem_ld16_issue(taddr(c + 1), rb);
          if (!process(c, ra)) { ok = false; tmem_ld_wait(rb); break; }
          tmem_ld_wait(rb);
          if (c + 2 < bw / 32) tmem_ld16_issue(taddr(c + 2), ra);
          if (!process(c + 1, rb)) {
            ok = false;
            if (c + 2 < bw / 32) tmem_ld_wait(ra);
            break;
          }
        }
        if (!ok) break;
      } else {
        const int CH = bw / 64;          // 32-column chunks per warp
        // the stage as a compile-time constant: each instantiation keeps only its own context live
        t.xs = xpose + (warp - 2) * (32 * 33);
        auto chunks = [&](auto tag) {
          constexpr int kSt = decltype(tag)::value;
#pragma unroll 1
          for (int ch = half * CH; ch < (half + 1) * CH; ++ch) {
            float v[32];
            tmem_ld32(tmem_base + (uint32_t)(acc * kBN + ch * 32) + ((uint32_t)(ew * 32) << 16), v);
            epi_chunk<32, kSt>(t, tm * BM + lrow, cbase + ch * 32, v, &pacc);
          }
        };
        switch (stage) {
          case ST_GRAM: chunks(StageTag<ST_GRAM>{}); break;
          case ST_POLY: chunks(StageTag<ST_POLY>{}); break;
          case ST_AXPY: chunks(StageTag<ST_AXPY>{}); break;
          case ST_QAXPY: chunks(StageTag<ST_QAXPY>{}); break;
          case ST_REUSE: chunks(StageTag<ST_REUSE>{}); break;
          case ST_PROBE: chunks(StageTag<ST_PROBE>{}); break;
          case ST_AA1: chunks(StageTag<ST_AA1>{}); break;
          case ST_AA2: chunks(StageTag<ST_AA2>{}); break;
          default: chunks(StageTag<ST_QX>{}); break;
        }
      }
      fence_before();
      if constexpr (kPair) {
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(at_rank0(tempty_bar + 8 * acc));
      } else {
        mbar_arrive_relaxed(tempty_bar + 8 * acc);
      }
      if (!kSrc && stage == ST_PROBE) {  // one partial per epilogue warp: no barrier, fixed order later
#pragma unroll
        for (int o2 = 16; o2 > 0; o2 >>= 1) pacc += __shfl_xor_sync(0xffffffffu, pacc, o2);
        if (lane == 0) {  // slots 0..7: the even (or only) CTA's warps, 8..15: the odd CTA's (zero on one SM)
          h.probe_partials[kProbeSlots * tiles[i] + (warp - 2) + 8 * (int)rank] = pacc;
          if (!kPair) h.probe_partials[kProbeSlots * tiles[i] + (warp - 2) + 8] = 0.f;
        }
      }
      if (++acc == 2) { acc = 0; acc_ph ^= 1u; }
    }
    if (!ok) {
      *abort_flag = 1;
      if (h.status) atomicOr(h.status, SMUON_DEV_WAIT_TIMEOUT);
    }
  }
  fence_before();
  if constexpr (kPair) {
    __syncwarp();
    cluster_sync_all();  // neither CTA leaves (or frees TMEM) while the other may still signal it
  } else {
    __syncthreads();
  }
  fence_after();
  if (warp == 1) {
    if constexpr (kPair) asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(C::TMEM_COLS));
    else asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(C::TMEM_COLS));
  }
}

template <bool kSplit, int kBN, bool kShallow, bool kSrc>
__global__ void __launch_bounds__(Cfg<kSplit, kBN, kShallow, kSrc>::NTHREADS, 1)
    k_gemm_tc(const Plan* plan, int stage, int iter, const int32_t* skip) {
  if (skip && *skip) return;
  gemm_tc_body<kSplit, kBN, kShallow, kSrc, false>(plan, stage, iter);
}

// SM pairs: 256 x 256 tiles, one cluster of two CTAs per pair of SMs
template <bool kSplit, bool kShallow, bool kSrc>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(Cfg<kSplit, 256, kShallow, kSrc, true>::NTHREADS, 1)
    k_gemm_tc2(const Plan* plan, int stage, int iter, const int32_t* skip) {
  if (skip && *skip) return;  // read by both CTAs of a pair: both leave, or neither
  gemm_tc_body<kSplit, 256, kShallow, kSrc, true>(plan, stage, iter);
}

}  // namespace tc

template <bool kSplit, int kBN, bool kShallow, bool kSrc, bool kPair>
static cudaError_t launch_tc_variant(const Plan* d_plan, int stage, int iter, const int32_t* skip, int grid,
                                     cudaStream_t s) {
  using C = tc::Cfg<kSplit, kBN, kShallow, kSrc, kPair>;
  static bool attr_set[256] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if constexpr (kPair) {
    if (dev < 256 && !attr_set[dev]) {
      cudaError_t e = cudaFuncSetAttribute(tc::k_gemm_tc2<kSplit, kShallow, kSrc>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
      if (e != cudaSuccess) return e;
      attr_set[dev] = true;
    }
    // grid = the pairs' CTAs (a multiple of the cluster size)
    tc::k_gemm_tc2<kSplit, kShallow, kSrc><<<2 * grid, C::NTHREADS, C::SMEM_BYTES, s>>>(d_plan, stage, iter, skip);
  } else {
    if (dev < 256 && !attr_set[dev]) {
      cudaError_t e = cudaFuncSetAttribute(tc::k_gemm_tc<kSplit, kBN, kShallow, kSrc>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
      if (e != cudaSuccess) return e;
      attr_set[dev] = true;
    }
    tc::k_gemm_tc<kSplit, kBN, kShallow, kSrc><<<grid, C::NTHREADS, C::SMEM_BYTES, s>>>(d_plan, stage, iter, skip);
  }
  return cudaGetLastError();
}

template <bool kSplit, int kBN, bool kSrc, bool kPair>
static cudaError_t launch_tc_src(const PlanHeader& h, const Plan* d_plan, int stage, int iter,
                                 const int32_t* skip, int grid, cudaStream_t s) {
  // split operands of 256-wide single-SM tiles take 96 KB per ring stage: only the deep ring holds two
  if (h.max_k[stage] <= kShallowMaxK && !(kSplit && kBN == 256 && !kPair))
    return launch_tc_variant<kSplit, kBN, true, kSrc, kPair>(d_plan, stage, iter, skip, grid, s);
  return launch_tc_variant<kSplit, kBN, false, kSrc, kPair>(d_plan, stage, iter, skip, grid, s);
}

template <bool kSplit, int kBN, bool kPair>
static cudaError_t launch_tc_depth(const PlanHeader& h, const Plan* d_plan, int stage, int iter,
                                   const int32_t* skip, int grid, cudaStream_t s) {
  // the B X stage takes its X source through the shared-memory ring when the plan has the maps and
  // runs several steps (measured: with a single step the direct loads of the row-per-lane epilogue,
  // served by L1, were 4% faster on the ResNet-50 set; from two steps on the ring wins, 5-12%)
  if (stage == ST_AXPY && h.axpy_tma && h.iters >= 2)
    return launch_tc_src<kSplit, kBN, true, kPair>(h, d_plan, stage, iter, skip, grid, s);
  return launch_tc_src<kSplit, kBN, false, kPair>(h, d_plan, stage, iter, skip, grid, s);
}

int tc_tile_n(int stage, uint32_t flags) {
  (void)stage;
  return (flags & SMUON_NS_SPLIT_BF16) ? kSplitBN : 256;  // split mode needs the smem for its lo tiles
}

int tc_pair_clusters() {
  // pairs of SMs that can hold one cluster of the pair kernel each (its largest shared-memory form);
  // the GPCs need not split evenly into pairs
  static int cached[256] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (dev < 256 && cached[dev] > 0) return cached[dev];
  using C = tc::Cfg<true, 256, false, true, true>;
  auto fn = tc::k_gemm_tc2<true, false, true>;
  if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES) != cudaSuccess) return 0;
  int sms = 0;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * (sms / 2), 1, 1);
  cfg.blockDim = dim3(C::NTHREADS, 1, 1);
  cfg.dynamicSmemBytes = C::SMEM_BYTES;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, (const void*)fn, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  if (dev < 256) cached[dev] = n;
  return n;
}

cudaError_t launch_gemm_tc(const Plan* d_plan, const PlanHeader& h, int stage, int iter, const int32_t* skip,
                           int num_sms, cudaStream_t s) {
  (void)num_sms;  // the plan's schedule fixed the grid: one CTA (or pair) per scheduled tile list
  const int grid = h.sched_ctas[stage];
  if (h.total_tiles[stage] == 0 || grid <= 0) return cudaSuccess;
  const bool split = (h.flags & SMUON_NS_SPLIT_BF16) && split_stage(stage);
  if (h.pair) {
    if (split) return launch_tc_depth<true, 256, true>(h, d_plan, stage, iter, skip, grid, s);
    return launch_tc_depth<false, 256, true>(h, d_plan, stage, iter, skip, grid, s);
  }
  if (split) return launch_tc_depth<true, kSplitBN, false>(h, d_plan, stage, iter, skip, grid, s);
  if (tc_tile_n(stage, h.flags) == 128) return launch_tc_depth<false, 128, false>(h, d_plan, stage, iter, skip, grid, s);
  return launch_tc_depth<false, 256, false>(h, d_plan, stage, iter, skip, grid, s);
}

}  // namespace smuon
