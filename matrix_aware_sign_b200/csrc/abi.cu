// abi.cu -- host side of the C ABI declared in include/smuon.h.
//
// Checks arguments before enqueueing anything, lays out the caller's
// workspace, builds the device plan (groups, per-matrix descriptors, TMA
// tensor maps, tile tables), uploads it with a kernel and launches the
// stage kernels on the caller's stream. The host never reads device data.
#include <algorithm>
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <functional>
#include <map>
#include <memory>
#include <mutex>
#include <queue>
#include <string>
#include <vector>

#include "epilogue.cuh"

using namespace smuon;

namespace {

thread_local std::string g_err;

smuon_status fail(smuon_status code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_err = buf;
  return code;
}

#define CUDA_TRY(expr)                                                                  \
  do {                                                                                  \
    cudaError_t e_ = (expr);                                                            \
    if (e_ != cudaSuccess)                                                              \
      return fail(SMUON_ERR_CUDA, "%s failed: %s", #expr, cudaGetErrorString(e_));      \
  } while (0)

// ------------------------------------------------------------------ launch trace
// Every kernel launch goes through a Launch guard: it counts the launch and,
// while tracing is on, brackets it with CUDA events on the launch stream and
// records the launch's algorithmic work (flops or bytes) for roofline reports.
struct TraceRec {
  const char* name;
  int32_t kind;
  double work;      // issued work (flops the tensor cores executed, or bytes)
  double nominal;   // the method's nominal count (equal to work for byte counts)
  cudaEvent_t a, b;
};

std::mutex g_tr_mu;
bool g_tr_on = false;
std::vector<TraceRec> g_tr;
std::vector<std::pair<cudaEvent_t, cudaEvent_t>> g_ev_free;
std::atomic<long long> g_launches{0};

struct Launch {
  TraceRec r{};
  bool on = false;
  cudaStream_t s;
  Launch(const char* name, int32_t kind, double work, cudaStream_t st, double nominal = -1.0) : s(st) {
    g_launches.fetch_add(1);
    std::lock_guard<std::mutex> lk(g_tr_mu);
    if (!g_tr_on || g_tr.size() >= 1000000) return;
    r.name = name; r.kind = kind; r.work = work; r.nominal = nominal < 0 ? work : nominal;
    if (!g_ev_free.empty()) {
      r.a = g_ev_free.back().first; r.b = g_ev_free.back().second;
      g_ev_free.pop_back();
    } else if (cudaEventCreate(&r.a) != cudaSuccess || cudaEventCreate(&r.b) != cudaSuccess) {
      return;
    }
    on = true;
    cudaEventRecord(r.a, s);
  }
  ~Launch() {
    if (!on) return;
    cudaEventRecord(r.b, s);
    std::lock_guard<std::mutex> lk(g_tr_mu);
    g_tr.push_back(r);
  }
};

// ------------------------------------------------------------------ device info
struct DevInfo {
  int sms = 0;
  int major = 0, minor = 0;
  bool ok = false;
};

std::mutex g_dev_mu;
std::map<int, DevInfo> g_dev;

smuon_status device_info(DevInfo* out) {
  int dev = 0;
  CUDA_TRY(cudaGetDevice(&dev));
  std::lock_guard<std::mutex> lk(g_dev_mu);
  auto it = g_dev.find(dev);
  if (it == g_dev.end()) {
    DevInfo d;
    CUDA_TRY(cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev));
    CUDA_TRY(cudaDeviceGetAttribute(&d.major, cudaDevAttrComputeCapabilityMajor, dev));
    CUDA_TRY(cudaDeviceGetAttribute(&d.minor, cudaDevAttrComputeCapabilityMinor, dev));
    d.ok = (d.major == 10 && d.minor == 0);
    it = g_dev.emplace(dev, d).first;
  }
  *out = it->second;
  if (!out->ok)
    return fail(SMUON_ERR_UNSUPPORTED, "device %d is sm_%d%d; this library is built for sm_100a only", dev,
                out->major, out->minor);
  return SMUON_OK;
}

// ------------------------------------------------------------------ tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

smuon_status get_encoder(EncodeTiledFn* fn) {
  static EncodeTiledFn cached = nullptr;
  static std::once_flag once;
  static cudaError_t err = cudaSuccess;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    err = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q);
    if (err == cudaSuccess && q == cudaDriverEntryPointSuccess) cached = reinterpret_cast<EncodeTiledFn>(p);
  });
  if (!cached) return fail(SMUON_ERR_CUDA, "cuTensorMapEncodeTiled is not available (%s)", cudaGetErrorString(err));
  *fn = cached;
  return SMUON_OK;
}

// 3-D bf16 map over [count][rows][ld] with box {box0 (inner), box1, 1}, 128B swizzle
smuon_status encode_bf16_3d(CUtensorMap* out, const void* ptr, int64_t inner, int64_t rows, int64_t count,
                            int64_t ld, uint32_t box0, uint32_t box1,
                            CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B) {
  EncodeTiledFn enc;
  smuon_status st = get_encoder(&enc);
  if (st != SMUON_OK) return st;
  cuuint64_t dims[3] = {(cuuint64_t)inner, (cuuint64_t)rows, (cuuint64_t)count};
  cuuint64_t strides[2] = {(cuuint64_t)(ld * 2), (cuuint64_t)(ld * 2 * rows)};
  cuuint32_t box[3] = {box0, box1, 1};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = enc(out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(SMUON_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return SMUON_OK;
}

// float32 3-D map (B X epilogue source): 128-byte swizzle for 32-float-wide boxes, none for wider ones
smuon_status encode_f32_3d(CUtensorMap* out, const void* ptr, int64_t inner, int64_t rows, int64_t count,
                           int64_t ld, uint32_t box0, uint32_t box1) {
  EncodeTiledFn enc;
  smuon_status st = get_encoder(&enc);
  if (st != SMUON_OK) return st;
  cuuint64_t dims[3] = {(cuuint64_t)inner, (cuuint64_t)rows, (cuuint64_t)count};
  cuuint64_t strides[2] = {(cuuint64_t)(ld * 4), (cuuint64_t)(ld * 4 * rows)};
  cuuint32_t box[3] = {box0, box1, 1};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = enc(out, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(ptr), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, box0 * 4 == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(SMUON_ERR_CUDA, "cuTensorMapEncodeTiled (f32) failed (%d)", (int)r);
  return SMUON_OK;
}

// ------------------------------------------------------------------ validation
int dtype_size(int32_t dt) { return dt == SMUON_F32 ? 4 : dt == SMUON_BF16 ? 2 : dt == SMUON_I8 ? 1 : 0; }

smuon_status check_mat(const smuon_mat& m, const char* what, int i, bool allow_f32, bool allow_bf16,
                       bool allow_i8, bool allow_bits = false) {
  if (!m.data) return fail(SMUON_ERR_INVALID_ARG, "%s[%d].data is NULL", what, i);
  if (m.rows < 1 || m.cols < 1 || m.rows > 65536 || m.cols > 65536)
    return fail(SMUON_ERR_SHAPE, "%s[%d] has shape %dx%d (each side must be in 1..65536)", what, i, m.rows, m.cols);
  if (m.ld < m.cols) return fail(SMUON_ERR_SHAPE, "%s[%d].ld=%lld < cols=%d", what, i, (long long)m.ld, m.cols);
  const bool ok = (m.dtype == SMUON_F32 && allow_f32) || (m.dtype == SMUON_BF16 && allow_bf16) ||
                  (m.dtype == SMUON_I8 && allow_i8) || (m.dtype == SMUON_BITS && allow_bits);
  if (!ok) return fail(SMUON_ERR_DTYPE, "%s[%d] has an unsupported dtype %d", what, i, m.dtype);
  if (m.dtype == SMUON_BITS) {  // a packed message: flat words, no row stride
    if (m.ld != m.cols) return fail(SMUON_ERR_SHAPE, "%s[%d] is a 1-bit message: ld must equal cols", what, i);
    if (reinterpret_cast<uintptr_t>(m.data) % 16 != 0)
      return fail(SMUON_ERR_INVALID_ARG, "%s[%d] is a 1-bit message: data must be 16-byte aligned", what, i);
    return SMUON_OK;
  }
  if (reinterpret_cast<uintptr_t>(m.data) % dtype_size(m.dtype) != 0)
    return fail(SMUON_ERR_INVALID_ARG, "%s[%d].data is not aligned to its element size", what, i);
  return SMUON_OK;
}

bool same_shape(const smuon_mat& a, const smuon_mat& b) { return a.rows == b.rows && a.cols == b.cols; }

// ------------------------------------------------------------------ NS plan
struct NsRequest {
  const smuon_mat* M_in;
  const smuon_mat* U_out;
  int32_t n_mats;
  const smuon_mat* G;
  float beta, a, b, c;
  int32_t iters;
  float eps;
  uint32_t flags;
  const smuon_mat* Q_out;   // EMIT_Q outputs, or (probe) the user's cached Q
  bool probe;               // build the CacheMuon REUSE + PROBE plan instead of the NS chain
  float gamma;
};

struct Layout {
  size_t plan_bytes = 0, total = 0;
  size_t off_groups = 0, off_mats = 0, off_tmaps = 0;
  size_t off_partials = 0, off_scale = 0, off_probe = 0, off_mom_begin = 0;
  size_t off_sched = 0, off_sched_begin = 0;
  size_t off_lz_rows = 0, off_rscale = 0, off_lz = 0, off_lz_ab = 0, off_lz_act = 0;
  int n_tmaps = 0;
};

struct Builder {
  std::vector<GroupDesc> groups;
  std::vector<MatDesc> mats;
  std::vector<CUtensorMap> maps;
  std::vector<int32_t> sched, sched_begin;  // tensor-core tile schedule (filled when base is set)
  PlanHeader h{};
  Layout L;
  size_t cursor = 0;
  char* base = nullptr;  // device workspace base (nullptr while sizing)

  size_t take(size_t bytes) {
    cursor = (size_t)round_up((int64_t)cursor, 256);
    size_t o = cursor;
    cursor += bytes;
    return o;
  }
  template <class T>
  T* ptr_at(size_t off) {
    return base ? reinterpret_cast<T*>(base + off) : nullptr;
  }
};

Mode pick_mode(uint32_t flags) {
  if (flags & SMUON_NS_FP32_REF) return MODE_SIMT_F32;
  if (flags & SMUON_NS_SIMT_BF16) return MODE_SIMT_BF16;
  return MODE_TC_BF16;
}

// Tile schedule of one tensor-core stage. The stages whose K is the long side
// n (Gram, probe) mix tiles of very different lengths across groups (a 512 x
// 4608 Gram tile runs 72 k-blocks, a 64 x 576 one 9): there, longest
// processing time first -- tiles in decreasing cost (ties in tile order) each
// onto the CTA with the least work so far. Cost of a tile in units of one
// 64-deep k-block of MMAs: its k-blocks (three MMAs each in split mode) plus
// about eight for the epilogue of a full 128 x 256 tile, scaled by the share
// of the tile that lies inside the matrix. The other stages (K = m) keep the
// round-robin order, tile t on CTA t mod ctas: their tiles are short and
// epilogue-bound, so a count-balanced order does better than the cost model.
bool lpt_stage(int st) { return st == ST_GRAM || st == ST_PROBE; }

void schedule_stage(const std::vector<GroupDesc>& groups, int st, int total, int ctas, int bm, int bn, bool split,
                    int32_t* ids, int32_t* begin) {
  std::vector<std::vector<int32_t>> per(ctas);
  if (!lpt_stage(st)) {
    // a last partial wave of r tiles with 2r <= ctas goes out as 2r half tiles, one per list, so it takes half
    // a tile's time instead of a whole one (B X only: its right operand is MN-major, cut along the columns)
    const int r = total % ctas;
    const int whole = (half_tile_stage(st) && r > 0 && 2 * r <= ctas) ? total - r : total;
    for (int t = 0; t < whole; ++t) per[t % ctas].push_back(t);
    for (int t = whole; t < total; ++t)
      for (int side = 0; side < 2; ++side)
        per[2 * (t - whole) + side].push_back(kHalfTileFlag | (side ? kHalfTileSide : 0) | t);
  } else {
    std::vector<std::pair<double, int32_t>> cost_tile;  // (cost, tile)
    cost_tile.reserve(total);
    for (const GroupDesc& g : groups) {
      const int tiles = sym_stage(st) ? sym_start(g.tiles_m[st], g.tiles_n[st], bn / bm)
                                      : g.tiles_m[st] * g.tiles_n[st];
      const int K = (st == ST_GRAM || st == ST_PROBE) ? g.n : g.m;
      const int No = wide_out_stage(st) ? g.n : g.m;
      // per SM: a pair's SMs each take a 128-row half of the 256 x 256 tile
      const double kb = (double)((K + 63) / 64) * (split && split_stage(st) ? 3 : 1) * bn / 256.0;
      const double fill = (double)g.m * No / ((double)g.tiles_m[st] * bm * g.tiles_n[st] * bn);
      const double cost = kb + 8.0 * fill * bn / 256.0;
      for (int t = g.tile_begin[st]; t < g.tile_begin[st] + g.count * tiles; ++t) cost_tile.push_back({cost, t});
    }
    std::stable_sort(cost_tile.begin(), cost_tile.end(),
                     [](const auto& x, const auto& y) { return x.first > y.first; });
    // least-loaded CTA first (ties: lowest index)
    using Load = std::pair<double, int32_t>;
    std::priority_queue<Load, std::vector<Load>, std::greater<Load>> heap;
    for (int c = 0; c < ctas; ++c) heap.push({0.0, c});
    for (const auto& ct : cost_tile) {
      Load l = heap.top();
      heap.pop();
      per[l.second].push_back(ct.second);
      heap.push({l.first + ct.first, l.second});
    }
  }
  int pos = 0;
  for (int c = 0; c < ctas; ++c) {
    begin[c] = pos;
    for (int32_t t : per[c]) ids[pos++] = t;
  }
  begin[ctas] = pos;
}

// Builds groups, descriptors and the workspace layout. With base == nullptr it
// only sizes the workspace; otherwise it also fills device pointers and maps.
smuon_status build_plan(const NsRequest& rq, char* base, Builder* B) {
  B->base = base;
  const Mode mode = pick_mode(rq.flags);
  const bool bf = (mode != MODE_SIMT_F32);
  const bool tc = (mode == MODE_TC_BF16);
  const bool emit_q = (rq.flags & SMUON_NS_EMIT_Q) && !rq.probe;
  const bool gram_only = (rq.flags & SMUON_NS_GRAM_ONLY) && !rq.probe;
  const bool spectral = (rq.flags & SMUON_NS_SPECTRAL) && !rq.probe;
  const int K = rq.iters;
  const int BM = tc ? kTcBM : kSimtBM;
  const size_t esz = bf ? 2 : 4;
  // split BF16: operand buffers hold [hi parts of all matrices][lo parts of all matrices]
  const int parts = (tc && (rq.flags & SMUON_NS_SPLIT_BF16) && !rq.probe) ? 2 : 1;

  // group by wide shape, biggest first
  std::map<std::pair<int, int>, std::vector<int>> by_shape;
  for (int i = 0; i < rq.n_mats; ++i) {
    const smuon_mat& M = rq.M_in[i];
    by_shape[{std::min(M.rows, M.cols), std::max(M.rows, M.cols)}].push_back(i);
  }
  std::vector<std::pair<std::pair<int, int>, std::vector<int>>> order(by_shape.begin(), by_shape.end());
  std::stable_sort(order.begin(), order.end(), [](const auto& x, const auto& y) {
    return (int64_t)x.first.first * x.first.second > (int64_t)y.first.first * y.first.second;
  });

  B->groups.clear();
  B->mats.clear();
  B->maps.clear();
  int mom_tiles = 0;
  for (auto& kv : order) {
    GroupDesc g{};
    g.m = kv.first.first;
    g.n = kv.first.second;
    g.count = (int32_t)kv.second.size();
    g.first_mat = (int32_t)B->mats.size();
    g.ldn = round_up(g.n, 128);
    g.ldm = round_up(g.m, 128);
    for (int z = 0; z < g.count; ++z) {
      const int i = kv.second[z];
      const smuon_mat& M = rq.M_in[i];
      MatDesc d{};
      d.m_ptr = M.data; d.m_ld = M.ld; d.m_dtype = M.dtype;
      if (rq.G) { d.g_ptr = rq.G[i].data; d.g_ld = rq.G[i].ld; d.g_dtype = rq.G[i].dtype; }
      d.u_ptr = rq.U_out[i].data; d.u_ld = rq.U_out[i].ld; d.u_dtype = rq.U_out[i].dtype;
      if (rq.Q_out && (emit_q || rq.probe)) { d.q_ptr = rq.Q_out[i].data; d.q_ld = rq.Q_out[i].ld; }
      d.rows = M.rows; d.cols = M.cols; d.tall = M.rows > M.cols ? 1 : 0;
      auto rows16 = [](const void* p, int64_t ld, int32_t dt) {
        return p && reinterpret_cast<uintptr_t>(p) % 16 == 0 && (ld * dtype_size(dt)) % 16 == 0;
      };
      d.vec = 0;
      if (M.dtype != SMUON_I8 && rows16(d.m_ptr, d.m_ld, d.m_dtype)) d.vec |= 1;
      if (rows16(d.u_ptr, d.u_ld, d.u_dtype)) d.vec |= 2;
      if (rows16(d.q_ptr, d.q_ld, SMUON_BF16)) d.vec |= 4;
      if (M.dtype == SMUON_F32 && rows16(d.m_ptr, d.m_ld, SMUON_F32) && M.cols % 4 == 0 &&
          (!d.g_ptr || (d.g_dtype == SMUON_F32 && rows16(d.g_ptr, d.g_ld, SMUON_F32))))
        d.vec |= 8;
      d.group = (int32_t)B->groups.size();
      d.z = z;
      d.mom_tiles_c = ceil_div(M.cols, 64);
      d.mom_count = ceil_div(M.rows, 64) * d.mom_tiles_c;
      d.mom_begin = mom_tiles;
      mom_tiles += d.mom_count;
      B->mats.push_back(d);
    }
    B->groups.push_back(g);
  }
  // momentum tiles must be increasing along mats for the device binary search: they are.
  // spectral scaling: Lanczos vectors v_0 .. v_K and the work vector w of each matrix, m floats each
  int64_t lz_floats = 0;
  for (MatDesc& d : B->mats) {
    d.lz_off = lz_floats;
    if (spectral) lz_floats += (int64_t)(kLanczosSteps + 2) * lz_stride(B->groups[d.group].m);
  }

  // SM pairs (256 x 256 tiles over clusters of two CTAs) for every tensor-core stage when no matrix is too
  // small for a 256-row tile; decided from the flags and shapes alone, so the sizing pass and the filling
  // pass lay the workspace out alike
  bool pair = tc && !(rq.flags & SMUON_NS_ONE_SM);
  for (const auto& g : B->groups)
    if (g.m < kPairMinM) pair = false;
  const int TBM = pair ? 2 * kTcBM : BM;  // tile height of the tables

  // tile tables: for the symmetric stages the tiles that reach the diagonal or
  // lie above it (BN = ratio * TBM), a full grid of TBM x BN tiles otherwise
  int totals[ST_COUNT] = {0};
  int ratios[ST_COUNT] = {0};
  for (int st = 0; st < ST_COUNT; ++st) {
    const int BN = tc ? tc_tile_n(st, rq.flags) : kSimtBN;
    ratios[st] = BN / TBM;
  }
  for (auto& g : B->groups) {
    const int tmm = ceil_div(g.m, TBM);
    for (int st = 0; st < ST_COUNT; ++st) {
      const bool sym = sym_stage(st);
      const int BN = TBM * ratios[st];
      const int No = wide_out_stage(st) ? g.n : g.m;
      g.tiles_m[st] = tmm;
      g.tiles_n[st] = ceil_div(No, BN);
      g.tile_begin[st] = totals[st];
      if ((st == ST_AA1 || st == ST_AA2 || st == ST_QX) && !gram_only) continue;  // the Gram-only solve's own
      totals[st] += g.count * (sym ? sym_start(tmm, g.tiles_n[st], ratios[st]) : g.tiles_m[st] * g.tiles_n[st]);
    }
  }

  // tile schedule sizes (tensor-core mode): every tile id once, a begin array per stage
  int sched_off[ST_COUNT] = {0}, sched_boff[ST_COUNT] = {0};
  int sched_n = 0, begin_n = 0;
  for (int st = 0; st < ST_COUNT; ++st) {
    sched_off[st] = sched_n;
    sched_boff[st] = begin_n;
    if (!tc) continue;
    // a B X stage may list up to one extra entry per list (a tile of its last wave cut in two halves)
    sched_n += totals[st] + (half_tile_stage(st) ? std::min(totals[st], kMaxSchedCtas) : 0);
    begin_n += std::min(totals[st], kMaxSchedCtas) + 1;
  }

  // layout: plan region first
  Layout& L = B->L;
  B->cursor = 0;
  const size_t hdr = B->take(sizeof(Plan));
  (void)hdr;
  L.off_groups = B->take(sizeof(GroupDesc) * B->groups.size());
  L.off_mats = B->take(sizeof(MatDesc) * B->mats.size());
  L.off_mom_begin = B->take(sizeof(int32_t) * (B->mats.size() + 1));
  L.off_sched = B->take(sizeof(int32_t) * std::max(sched_n, 1));
  L.off_sched_begin = B->take(sizeof(int32_t) * std::max(begin_n, 1));
  L.off_lz_rows = B->take(sizeof(int32_t) * (B->mats.size() + 1));
  // the B X epilogue reads its X source through a TMA-fed shared-memory ring when every matrix's
  // momentum is f32 with 16-byte aligned rows (later steps read the workspace's copy of X, always aligned)
  bool axpy_tma = tc && !rq.probe && !gram_only;
  for (const MatDesc& d : B->mats)
    if (!(d.m_dtype == SMUON_F32 && reinterpret_cast<uintptr_t>(d.m_ptr) % 16 == 0 && (d.m_ld * 4) % 16 == 0))
      axpy_tma = false;
  // tensor maps: count them first
  auto want_map = [&](int32_t& slot) { slot = L.n_tmaps++; };
  L.n_tmaps = 0;
  for (auto& d : B->mats) {
    d.tm_src = -1;
    if (axpy_tma) want_map(d.tm_src);
  }
  for (auto& g : B->groups) {
    for (int i = 0; i < 2; ++i) {
      g.tm_x_k[i] = g.tm_x_mn[i] = g.tm_q_mn[i] = g.tm_x_kw[i] = g.tm_q_k[i] = g.tm_xf[i] = -1;
    }
    if (axpy_tma && bf && K >= 2) want_map(g.tm_xf[1]);
    if (axpy_tma && bf && K >= 3) want_map(g.tm_xf[0]);
    g.tm_a_k = g.tm_b_k = g.tm_uq_k = g.tm_a_kw = g.tm_t_k = g.tm_t_kw = -1;
    if (!tc) continue;
    const bool wide = !pair && tc_tile_n(ST_GRAM, rq.flags) == 256;  // a pair's CTAs stage 128-row B halves
    if (!rq.probe) {
      want_map(g.tm_x_k[0]);
      want_map(g.tm_x_mn[0]);
      if (wide) want_map(g.tm_x_kw[0]);
      if (gram_only) {  // T operand (right operand of B T) and Q_K as the left operand of Q_K X_0
        want_map(g.tm_t_k);
        if (wide) want_map(g.tm_t_kw);
        want_map(g.tm_q_k[K & 1]);
      }
      if (K >= 2 && !gram_only) {
        want_map(g.tm_x_k[1]);
        want_map(g.tm_x_mn[1]);
        if (wide) want_map(g.tm_x_kw[1]);
      }
      if (rq.c != 0.f) {
        want_map(g.tm_a_k);
        if (wide) want_map(g.tm_a_kw);
      }
      want_map(g.tm_b_k);
      if (emit_q && K >= 2) want_map(g.tm_q_mn[1]);
      if (emit_q && K >= 3) want_map(g.tm_q_mn[0]);
    } else {
      want_map(g.tm_x_mn[0]);
      want_map(g.tm_uq_k);
      want_map(g.tm_x_k[1]);
      if (wide) want_map(g.tm_x_kw[1]);
    }
  }
  L.off_tmaps = B->take(sizeof(CUtensorMap) * std::max(L.n_tmaps, 1));
  L.plan_bytes = (size_t)round_up((int64_t)B->cursor, 256);
  L.off_partials = B->take(sizeof(float) * kMomSlots * std::max(mom_tiles, 1));
  L.off_scale = B->take(sizeof(float) * B->mats.size());
  L.off_probe = B->take(sizeof(float) * kProbeSlots * std::max(totals[ST_PROBE], 1));
  L.off_rscale = B->take(sizeof(float) * B->mats.size());
  L.off_lz = spectral ? B->take(sizeof(float) * lz_floats) : 0;
  L.off_lz_ab = spectral ? B->take(sizeof(float) * 2 * kLanczosSteps * B->mats.size()) : 0;
  // the active list ([count][rows prefix][matrices]) and the step launches' ticket
  L.off_lz_act = spectral ? B->take(sizeof(int32_t) * (2 * B->mats.size() + 3)) : 0;

  // per-group buffers
  for (auto& g : B->groups) {
    const size_t nx = (size_t)g.count * g.m * g.ldn, nm = (size_t)g.count * g.m * g.ldm;
    g.xop[0] = B->ptr_at<void>(B->take(nx * esz * parts));
    g.xop[1] = nullptr;
    g.xf[0] = g.xf[1] = nullptr;
    g.af = nullptr; g.aop = nullptr; g.bop = nullptr;
    g.af2 = nullptr; g.aop2 = nullptr;
    g.qf[0] = g.qf[1] = nullptr; g.qop[0] = g.qop[1] = nullptr;
    if (rq.probe) {
      g.xop[1] = B->ptr_at<void>(B->take(nx * esz));
      continue;
    }
    if (gram_only) {  // no X iterates: T between the two updates of A instead
      g.af2 = B->ptr_at<float>(B->take(nm * 4));
      g.aop2 = B->ptr_at<void>(B->take(nm * 2 * parts));
    }
    if (K >= 2 && !gram_only) g.xop[1] = B->ptr_at<void>(B->take(nx * esz * parts));
    // f32 masters of X between steps: plain BF16 keeps one (its operand holds only bf16(X)); split mode
    // carries X as its hi and lo operand parts, which the B X epilogue reads back as hi + lo
    if (bf && parts == 1 && K >= 2 && !gram_only) g.xf[1] = B->ptr_at<float>(B->take(nx * 4));
    if (bf && parts == 1 && K >= 3 && !gram_only) g.xf[0] = B->ptr_at<float>(B->take(nx * 4));
    // f32 A: the Lanczos input (spectral scaling) and the Gram-only solve's A iterates read it; the b A term of
    // the A^2 stage reads A's hi + lo parts in split mode (so a CacheMuon fresh solve with the transform rounds
    // exactly as the plain chain does), the f32 A in the other modes
    const bool af_needed = spectral || gram_only || parts == 1;
    if ((rq.c != 0.f && af_needed) || spectral) g.af = B->ptr_at<float>(B->take(nm * 4));
    if (rq.c != 0.f) g.aop = bf ? B->ptr_at<void>(B->take(nm * 2 * parts)) : (void*)g.af;
    g.bop = B->ptr_at<void>(B->take(nm * esz * parts));
    if (emit_q && (K >= 2 || gram_only)) {
      g.qop[1] = B->ptr_at<void>(B->take(nm * esz * parts));
      g.qf[1] = bf ? B->ptr_at<float>(B->take(nm * 4)) : reinterpret_cast<float*>(g.qop[1]);
    }
    if (emit_q && (K >= 3 || (gram_only && K >= 2))) {
      g.qop[0] = B->ptr_at<void>(B->take(nm * esz * parts));
      g.qf[0] = bf ? B->ptr_at<float>(B->take(nm * 4)) : reinterpret_cast<float*>(g.qop[0]);
    }
  }
  L.total = (size_t)round_up((int64_t)B->cursor, 256);

  // header
  PlanHeader& h = B->h;
  h = PlanHeader{};
  h.n_mats = (int32_t)B->mats.size();
  h.n_groups = (int32_t)B->groups.size();
  h.n_tmaps = L.n_tmaps;
  h.mode = mode;
  h.iters = K;
  h.flags = rq.flags;
  h.a = rq.a; h.b = rq.b; h.c = rq.c; h.eps = rq.eps; h.beta = rq.beta; h.gamma = rq.gamma;
  h.total_mom_tiles = mom_tiles;
  // pipeline waits of the tensor-core stages: about 2 s of SM clock, or (failure-detection test) a
  // budget that runs out while the producer issues nothing
  h.wait_cycles = (rq.flags & SMUON_NS_TEST_WAIT_EXPIRY) ? (1ull << 16) : (1ull << 32);
  h.starve_tc = (rq.flags & SMUON_NS_TEST_WAIT_EXPIRY) ? 1 : 0;
  h.tile_bm = TBM; h.tile_bn = tc ? tc_tile_n(ST_AXPY, rq.flags) : kSimtBN;
  h.pair = pair ? 1 : 0;
  for (int st = 0; st < ST_COUNT; ++st) {
    h.total_tiles[st] = totals[st];
    h.sym_ratio[st] = ratios[st];
  }
  h.partials = B->ptr_at<float>(L.off_partials);
  h.scale = B->ptr_at<float>(L.off_scale);
  h.probe_partials = B->ptr_at<float>(L.off_probe);
  h.rscale = B->ptr_at<float>(L.off_rscale);
  h.lz = spectral ? B->ptr_at<float>(L.off_lz) : nullptr;
  h.lz_ab = spectral ? B->ptr_at<float>(L.off_lz_ab) : nullptr;
  h.lz_rows = B->ptr_at<int32_t>(L.off_lz_rows);
  h.lz_act = spectral ? B->ptr_at<int32_t>(L.off_lz_act) : nullptr;
  h.mom_begin = B->ptr_at<int32_t>(L.off_mom_begin);
  h.sched = B->ptr_at<int32_t>(L.off_sched);
  h.sched_begin = B->ptr_at<int32_t>(L.off_sched_begin);
  for (int st = 0; st < ST_COUNT; ++st) {
    h.sched_off[st] = sched_off[st];
    h.sched_boff[st] = sched_boff[st];
    h.sched_ctas[st] = 0;
    h.max_k[st] = 0;
    h.axpy_tma = axpy_tma ? 1 : 0;
    for (const GroupDesc& g : B->groups)
      h.max_k[st] = std::max(h.max_k[st], (st == ST_GRAM || st == ST_PROBE) ? g.n : g.m);
  }
  h.groups = B->ptr_at<GroupDesc>(L.off_groups);
  h.mats = B->ptr_at<MatDesc>(L.off_mats);
  h.tmaps = B->ptr_at<CUtensorMap>(L.off_tmaps);

  if (!base) return SMUON_OK;

  // tile schedules over this device's SMs (one persistent CTA per SM)
  B->sched.assign(std::max(sched_n, 1), 0);
  B->sched_begin.assign(std::max(begin_n, 1), 0);
  if (tc) {
    DevInfo di;
    smuon_status dst = device_info(&di);
    if (dst != SMUON_OK) return dst;
    const bool split = (rq.flags & SMUON_NS_SPLIT_BF16) != 0 && parts == 2;
    // one tile list per CTA, or per pair of SMs that the device holds at once
    const int lists = pair ? tc_pair_clusters() : di.sms;
    if (lists <= 0) return fail(SMUON_ERR_CUDA, "the device holds no cluster of the SM-pair GEMM kernel");
    for (int st = 0; st < ST_COUNT; ++st) {
      if (totals[st] == 0) continue;
      const int ctas = std::min(std::min(totals[st], lists), kMaxSchedCtas);
      h.sched_ctas[st] = ctas;
      schedule_stage(B->groups, st, totals[st], ctas, TBM, TBM * ratios[st], split,
                     B->sched.data() + sched_off[st], B->sched_begin.data() + sched_boff[st]);
    }
  }

  // tensor maps
  B->maps.assign(std::max(L.n_tmaps, 1), CUtensorMap{});
  for (auto& g : B->groups) {
    if (!tc) continue;
    // K-major boxes {64, rows} and MN-major boxes {64, 64}, both with the 128-byte swizzle
    auto enc = [&](int32_t slot, const void* p, int64_t inner, int64_t rows, int64_t cnt, int64_t ld,
                   uint32_t b1) -> smuon_status {  // K-major
      if (slot < 0) return SMUON_OK;
      return encode_bf16_3d(&B->maps[slot], p, inner, rows, cnt, ld, 64, b1);
    };
    auto enc_mn = [&](int32_t slot, const void* p, int64_t inner, int64_t rows, int64_t cnt,
                      int64_t ld) -> smuon_status {
      if (slot < 0) return SMUON_OK;
      return encode_bf16_3d(&B->maps[slot], p, inner, rows, cnt, ld, 64, 64);
    };
    smuon_status st;
    const int64_t zc = (int64_t)g.count * parts;  // matrices in the map: hi parts, then lo parts
    for (int i = 0; i < 2; ++i) {
      if ((st = enc(g.tm_x_k[i], g.xop[i], g.n, g.m, zc, g.ldn, 128)) != SMUON_OK) return st;
      if ((st = enc_mn(g.tm_x_mn[i], g.xop[i], g.n, g.m, zc, g.ldn)) != SMUON_OK) return st;
      if ((st = enc_mn(g.tm_q_mn[i], g.qop[i], g.m, g.m, zc, g.ldm)) != SMUON_OK) return st;
      if ((st = enc(g.tm_q_k[i], g.qop[i], g.m, g.m, zc, g.ldm, 128)) != SMUON_OK) return st;
      if ((st = enc(g.tm_x_kw[i], g.xop[i], g.n, g.m, zc, g.ldn, 256)) != SMUON_OK) return st;
    }
    if ((st = enc(g.tm_a_kw, g.aop, g.m, g.m, zc, g.ldm, 256)) != SMUON_OK) return st;
    if ((st = enc(g.tm_t_k, g.aop2, g.m, g.m, zc, g.ldm, 128)) != SMUON_OK) return st;
    if ((st = enc(g.tm_t_kw, g.aop2, g.m, g.m, zc, g.ldm, 256)) != SMUON_OK) return st;
    if ((st = enc(g.tm_a_k, g.aop, g.m, g.m, zc, g.ldm, 128)) != SMUON_OK) return st;
    if ((st = enc(g.tm_b_k, g.bop, g.m, g.m, zc, g.ldm, 128)) != SMUON_OK) return st;
    if (g.tm_uq_k >= 0) {
      const MatDesc& d = B->mats[g.first_mat];
      if ((st = encode_bf16_3d(&B->maps[g.tm_uq_k], d.q_ptr, g.m, g.m, 1, d.q_ld, 64, 128)) != SMUON_OK) return st;
    }
    for (int i = 0; i < 2; ++i) {  // the B X epilogue's source of X_i, 32 x 128 boxes
      if (g.tm_xf[i] < 0) continue;
      if (parts == 1)  // f32 master [count][m][ldn]
        st = encode_f32_3d(&B->maps[g.tm_xf[i]], g.xf[i], g.n, g.m, g.count, g.ldn, 32, 128);
      else  // bf16 hi parts then lo parts [2 count][m][ldn], 64-byte rows with the 64-byte swizzle
        st = encode_bf16_3d(&B->maps[g.tm_xf[i]], g.xop[i], g.n, g.m, zc, g.ldn, 32, 128, CU_TENSOR_MAP_SWIZZLE_64B);
      if (st != SMUON_OK) return st;
    }
  }
  for (const MatDesc& d : B->mats) {  // the momentum as the first B X step's source
    if (d.tm_src < 0) continue;
    smuon_status st = d.tall ? encode_f32_3d(&B->maps[d.tm_src], d.m_ptr, d.cols, d.rows, 1, d.m_ld, 128, 32)
                             : encode_f32_3d(&B->maps[d.tm_src], d.m_ptr, d.cols, d.rows, 1, d.m_ld, 32, 128);
    if (st != SMUON_OK) return st;
  }
  return SMUON_OK;
}

smuon_status upload_plan(Builder& B, cudaStream_t s) {
  std::vector<unsigned char> bytes(B.L.plan_bytes, 0);
  Plan p;
  p.h = B.h;
  memcpy(bytes.data(), &p, sizeof(Plan));
  memcpy(bytes.data() + B.L.off_groups, B.groups.data(), sizeof(GroupDesc) * B.groups.size());
  memcpy(bytes.data() + B.L.off_mats, B.mats.data(), sizeof(MatDesc) * B.mats.size());
  {
    std::vector<int32_t> mb(B.mats.size() + 1);
    for (size_t i = 0; i < B.mats.size(); ++i) mb[i] = B.mats[i].mom_begin;
    mb[B.mats.size()] = B.h.total_mom_tiles;
    memcpy(bytes.data() + B.L.off_mom_begin, mb.data(), sizeof(int32_t) * mb.size());
  }
  memcpy(bytes.data() + B.L.off_sched, B.sched.data(), sizeof(int32_t) * B.sched.size());
  {  // first row of each matrix's A in the flattened row space of the Lanczos products
    std::vector<int32_t> lr(B.mats.size() + 1, 0);
    for (size_t i = 0; i < B.mats.size(); ++i) lr[i + 1] = lr[i] + B.groups[B.mats[i].group].m;
    memcpy(bytes.data() + B.L.off_lz_rows, lr.data(), sizeof(int32_t) * lr.size());
  }
  memcpy(bytes.data() + B.L.off_sched_begin, B.sched_begin.data(), sizeof(int32_t) * B.sched_begin.size());
  if (B.L.n_tmaps > 0) memcpy(bytes.data() + B.L.off_tmaps, B.maps.data(), sizeof(CUtensorMap) * B.L.n_tmaps);
  static UploadChunk chunk;  // large parameter block; filled then launched by value
  static std::mutex mu;
  std::lock_guard<std::mutex> lk(mu);
  for (size_t off = 0; off < bytes.size(); off += kUploadBytes) {
    const size_t n = std::min(bytes.size() - off, (size_t)kUploadBytes);
    chunk.dst = B.base + off;
    chunk.bytes = (int32_t)n;
    memcpy(chunk.data, bytes.data() + off, n);
    const int blocks = (int)std::min<size_t>(8, (n / 16 + 255) / 256);
    Launch L("k_plan_upload", SMUON_WORK_BYTES, 2.0 * n, s);
    k_plan_upload<<<std::max(blocks, 1), 256, 0, s>>>(chunk);
    CUDA_TRY(cudaGetLastError());
  }
  return SMUON_OK;
}

// algorithmic flops of one stage over the whole batch: 2 * Mo * No * K per matrix
double stage_flops(const Builder& B, int st) {
  double f = 0;
  for (const GroupDesc& g : B.groups) {
    const double m = g.m, n = g.n;
    double per = 0;
    switch (st) {
      case ST_GRAM: case ST_PROBE: per = 2 * m * m * n; break;
      case ST_AXPY: case ST_REUSE: case ST_QX: per = 2 * m * n * m; break;
      default: per = 2 * m * m * m; break;
    }
    f += per * g.count;
  }
  return f;
}

// flops the tensor cores (or CUDA cores) actually execute for a stage: tiles
// x 2 * BM * BN * (K rounded up to the k-block), three products in split mode
double stage_issued(const Builder& B, int st, int iter = 1 << 20) {
  const PlanHeader& h = B.h;
  const bool tc = h.mode == MODE_TC_BF16;
  const int BM = tc ? h.tile_bm : kSimtBM, BK = tc ? 64 : 16;
  const bool split = tc && (h.flags & SMUON_NS_SPLIT_BF16) && split_stage(st);
  double f = 0;
  for (const GroupDesc& g : B.groups) {
    // split mode: three products per tile, one in a group's plain leading steps
    const double parts = !split ? 1.0 : (plain_lead_stage(h.flags, st, iter, g.m) ? 1.0 : 3.0);
    const bool sym = sym_stage(st);
    const int BN = sym ? BM : (tc ? tc_tile_n(st, h.flags) : kSimtBN);
    const int T = g.tiles_m[st];
    const double tiles = (double)g.count * (sym ? T * (T + 1) / 2 : T * g.tiles_n[st]);
    const int K = (st == ST_GRAM || st == ST_PROBE) ? g.n : g.m;
    const double kpad = (double)((K + BK - 1) / BK) * BK;
    f += parts * tiles * 2.0 * BM * BN * kpad;
  }
  return f;
}

// algorithmic bytes of the momentum / normalisation prologue
double momentum_bytes(const NsRequest& rq, const PlanHeader& h) {
  double b = 0;
  const int op = (h.mode == MODE_SIMT_F32) ? 4 : ((h.flags & SMUON_NS_SPLIT_BF16) ? 4 : 2);
  for (int i = 0; i < rq.n_mats; ++i) {
    const double n = (double)rq.M_in[i].rows * rq.M_in[i].cols;
    b += n * dtype_size(rq.M_in[i].dtype) + n * op;
    if (rq.G) b += n * (dtype_size(rq.G[i].dtype) + 4);
  }
  return b;
}

smuon_status launch_gemm(const Plan* d_plan, const PlanHeader& h, int st, int iter, const int32_t* skip,
                         const DevInfo& di, cudaStream_t s, double stage_flops, double issued_flops) {
  const int total = h.total_tiles[st];
  if (total == 0) return SMUON_OK;
  // trace names: kernel, then the stage after a dot
  static const char* tc_names[2][ST_COUNT] = {
      {"k_gemm_tc.gram", "k_gemm_tc.poly", "k_gemm_tc.axpy", "k_gemm_tc.qaxpy", "k_gemm_tc.reuse", "k_gemm_tc.probe",
       "k_gemm_tc.aa1", "k_gemm_tc.aa2", "k_gemm_tc.qx"},
      {"k_gemm_tc_split.gram", "k_gemm_tc_split.poly", "k_gemm_tc_split.axpy", "k_gemm_tc_split.qaxpy",
       "k_gemm_tc_split.reuse", "k_gemm_tc_split.probe", "k_gemm_tc_split.aa1", "k_gemm_tc_split.aa2",
       "k_gemm_tc_split.qx"}};
  static const char* tc2_names[2][ST_COUNT] = {
      {"k_gemm_tc2.gram", "k_gemm_tc2.poly", "k_gemm_tc2.axpy", "k_gemm_tc2.qaxpy", "k_gemm_tc2.reuse",
       "k_gemm_tc2.probe", "k_gemm_tc2.aa1", "k_gemm_tc2.aa2", "k_gemm_tc2.qx"},
      {"k_gemm_tc2_split.gram", "k_gemm_tc2_split.poly", "k_gemm_tc2_split.axpy", "k_gemm_tc2_split.qaxpy",
       "k_gemm_tc2_split.reuse", "k_gemm_tc2_split.probe", "k_gemm_tc2_split.aa1", "k_gemm_tc2_split.aa2",
       "k_gemm_tc2_split.qx"}};
  if (h.mode == MODE_TC_BF16) {
    const bool split = (h.flags & SMUON_NS_SPLIT_BF16) && split_stage(st);
    const char* name = h.pair ? tc2_names[split][st] : tc_names[split][st];
    Launch L(name, SMUON_WORK_FLOPS, issued_flops, s, stage_flops);
    CUDA_TRY(launch_gemm_tc(d_plan, h, st, iter, skip, di.sms, s));
  } else {
    const int grid = std::min(total, di.sms * 6);
    Launch L(h.mode == MODE_SIMT_F32 ? "k_gemm_simt_f32" : "k_gemm_simt_bf16", SMUON_WORK_FLOPS, issued_flops, s,
             stage_flops);
    if (h.mode == MODE_SIMT_F32) k_gemm_simt_f32<<<grid, 256, 0, s>>>(d_plan, st, iter, skip);
    else k_gemm_simt_bf16<<<grid, 256, 0, s>>>(d_plan, st, iter, skip);
    CUDA_TRY(cudaGetLastError());
  }
  return SMUON_OK;
}

smuon_status validate_ns(const NsRequest& rq) {
  if (rq.n_mats < 1 || rq.n_mats > 4096) return fail(SMUON_ERR_INVALID_ARG, "n_mats=%d must be in 1..4096", rq.n_mats);
  if (!rq.M_in || !rq.U_out) return fail(SMUON_ERR_INVALID_ARG, "M_in and U_out must not be NULL");
  if (rq.iters < 1 || rq.iters > 64) return fail(SMUON_ERR_INVALID_ARG, "iters=%d must be in 1..64", rq.iters);
  const uint32_t known =
      SMUON_NS_FP32_REF | SMUON_NS_SPLIT_BF16 | SMUON_NS_NO_NORMALIZE | SMUON_NS_EMIT_Q | SMUON_NS_SIMT_BF16 |
      SMUON_NS_GRAM_ONLY | SMUON_NS_SPECTRAL | SMUON_NS_PLAIN_LEAD_MASK | SMUON_NS_TEST_WAIT_EXPIRY |
      SMUON_NS_ONE_SM;
  if (rq.flags & ~known) return fail(SMUON_ERR_INVALID_ARG, "unknown flag bits 0x%x", rq.flags & ~known);
  const uint32_t modes = rq.flags & (SMUON_NS_FP32_REF | SMUON_NS_SPLIT_BF16 | SMUON_NS_SIMT_BF16);
  if (modes & (modes - 1))
    return fail(SMUON_ERR_INVALID_ARG, "SMUON_NS_FP32_REF, SMUON_NS_SPLIT_BF16 and SMUON_NS_SIMT_BF16 are exclusive");
  if ((rq.flags & SMUON_NS_EMIT_Q) && !rq.Q_out)
    return fail(SMUON_ERR_INVALID_ARG, "SMUON_NS_EMIT_Q needs Q_out");
  if (rq.flags & SMUON_NS_GRAM_ONLY) {
    if (!(rq.flags & SMUON_NS_EMIT_Q))
      return fail(SMUON_ERR_INVALID_ARG, "SMUON_NS_GRAM_ONLY needs SMUON_NS_EMIT_Q (U = Q_K X_0)");
    if (rq.flags & (SMUON_NS_FP32_REF | SMUON_NS_SIMT_BF16))
      return fail(SMUON_ERR_UNSUPPORTED, "SMUON_NS_GRAM_ONLY runs on the tensor cores only");
    if (rq.n_mats != 1) return fail(SMUON_ERR_UNSUPPORTED, "SMUON_NS_GRAM_ONLY takes one matrix per call");
    if (rq.c == 0.f) return fail(SMUON_ERR_UNSUPPORTED, "SMUON_NS_GRAM_ONLY needs c != 0");
  }
  if ((rq.flags & SMUON_NS_SPECTRAL) && (rq.flags & (SMUON_NS_NO_NORMALIZE | SMUON_NS_EMIT_Q | SMUON_NS_GRAM_ONLY)))
    return fail(SMUON_ERR_UNSUPPORTED,
                "SMUON_NS_SPECTRAL excludes SMUON_NS_NO_NORMALIZE, SMUON_NS_EMIT_Q and SMUON_NS_GRAM_ONLY");
  if (rq.flags & SMUON_NS_PLAIN_LEAD_MASK) {
    if (!(rq.flags & SMUON_NS_SPLIT_BF16))
      return fail(SMUON_ERR_INVALID_ARG, "SMUON_NS_PLAIN_LEAD needs SMUON_NS_SPLIT_BF16");
    if (rq.flags & (SMUON_NS_SPECTRAL | SMUON_NS_EMIT_Q | SMUON_NS_GRAM_ONLY))
      return fail(SMUON_ERR_UNSUPPORTED,
                  "SMUON_NS_PLAIN_LEAD excludes SMUON_NS_SPECTRAL, SMUON_NS_EMIT_Q and SMUON_NS_GRAM_ONLY");
  }
  for (int i = 0; i < rq.n_mats; ++i) {
    smuon_status st;
    const bool has_g = rq.G != nullptr;
    if ((st = check_mat(rq.M_in[i], "M_in", i, true, !has_g, !has_g)) != SMUON_OK) return st;
    if ((st = check_mat(rq.U_out[i], "U_out", i, true, true, true, true)) != SMUON_OK) return st;
    if (!same_shape(rq.M_in[i], rq.U_out[i])) return fail(SMUON_ERR_SHAPE, "U_out[%d] shape differs from M_in", i);
    if (rq.U_out[i].dtype == SMUON_BITS) {
      if (rq.flags & (SMUON_NS_FP32_REF | SMUON_NS_SIMT_BF16))
        return fail(SMUON_ERR_UNSUPPORTED, "1-bit outputs need the tensor-core modes");
      if (rq.flags & (SMUON_NS_EMIT_Q | SMUON_NS_GRAM_ONLY))
        return fail(SMUON_ERR_UNSUPPORTED, "1-bit outputs are not written with SMUON_NS_EMIT_Q");
      if (rq.U_out[i].cols % 32 != 0)
        return fail(SMUON_ERR_SHAPE, "U_out[%d]: a 1-bit output needs cols %% 32 == 0 (cols=%d)", i,
                    rq.U_out[i].cols);
    }
    if (has_g) {
      if ((st = check_mat(rq.G[i], "G", i, true, true, false)) != SMUON_OK) return st;
      if (!same_shape(rq.M_in[i], rq.G[i])) return fail(SMUON_ERR_SHAPE, "G[%d] shape differs from M_in", i);
    }
    if (rq.flags & SMUON_NS_EMIT_Q) {
      const int m = std::min(rq.M_in[i].rows, rq.M_in[i].cols);
      if ((st = check_mat(rq.Q_out[i], "Q_out", i, false, true, false)) != SMUON_OK) return st;
      if (rq.Q_out[i].rows != m || rq.Q_out[i].cols != m)
        return fail(SMUON_ERR_SHAPE, "Q_out[%d] must be %dx%d", i, m, m);
    }
  }
  return SMUON_OK;
}

smuon_status check_ws(void* ws, size_t ws_bytes, size_t need) {
  if (!ws) return fail(SMUON_ERR_WORKSPACE, "workspace is NULL (need %zu bytes)", need);
  if (reinterpret_cast<uintptr_t>(ws) % 256 != 0) return fail(SMUON_ERR_WORKSPACE, "workspace must be 256-byte aligned");
  if (ws_bytes < need) return fail(SMUON_ERR_WORKSPACE, "workspace has %zu bytes, need %zu", ws_bytes, need);
  return SMUON_OK;
}

// enqueue the whole momentum + NS chain for a validated request
// everything the host needs to launch the kernels of a plan that is already in the workspace
struct NsExec {
  PlanHeader h;
  DevInfo di;
  const Plan* d_plan = nullptr;
  int iters = 1;
  float c = 0.f;
  uint32_t flags = 0;
  double mom_bytes = 0;
  double sflops[ST_COUNT] = {0};
  double sissued[ST_COUNT] = {0};
  double sissued_lead[8][ST_COUNT] = {{0}};  // issued flops of iteration k < 8 (plain leading steps)
  int64_t lz_rows = 0;          // spectral scaling: rows of all A_0 together
  double lz_matvec_bytes = 0;   // bytes of one A v product over the batch
};

smuon_status prepare_ns(const NsRequest& rq, void* ws, size_t ws_bytes, int32_t* d_status, cudaStream_t s,
                        NsExec* ex) {
  smuon_status st = device_info(&ex->di);
  if (st != SMUON_OK) return st;
  Builder B;
  if ((st = build_plan(rq, nullptr, &B)) != SMUON_OK) return st;
  if ((st = check_ws(ws, ws_bytes, B.L.total)) != SMUON_OK) return st;
  if ((st = build_plan(rq, reinterpret_cast<char*>(ws), &B)) != SMUON_OK) return st;
  B.h.status = d_status;
  if ((st = upload_plan(B, s)) != SMUON_OK) return st;
  ex->h = B.h;
  ex->d_plan = reinterpret_cast<const Plan*>(ws);
  ex->iters = rq.iters;
  ex->c = rq.c;
  ex->flags = rq.flags;
  ex->mom_bytes = momentum_bytes(rq, B.h);
  for (const MatDesc& d : B.mats) {
    const int m = B.groups[d.group].m;
    ex->lz_rows += m;
    const double a_bytes = (B.h.mode != MODE_SIMT_F32 && rq.c != 0.f && !(rq.flags & SMUON_NS_SPLIT_BF16))
                               ? 2.0 : 4.0;  // bf16 operand copy or f32 A
    ex->lz_matvec_bytes += a_bytes * m * m + 8.0 * m;
  }
  for (int k = 0; k < ST_COUNT; ++k) {
    ex->sflops[k] = stage_flops(B, k);
    ex->sissued[k] = stage_issued(B, k);
    for (int it = 0; it < 8; ++it) ex->sissued_lead[it][k] = stage_issued(B, k, it);
  }
  return SMUON_OK;
}

// spectral scaling: largest eigenvalue of each A_0 by Lanczos, then r = 1/(sqrt(lambda) + eps s)
smuon_status run_lanczos(const NsExec& ex, const int32_t* skip, cudaStream_t s) {
  const PlanHeader& h = ex.h;
  const int sms = ex.di.sms;
  const int mat_grid = std::max(1, std::min(h.n_mats, sms * 4));
  {
    Launch L("k_lz_start", SMUON_WORK_BYTES, 4.0 * ex.lz_rows, s);
    k_lz_start<<<mat_grid, 256, 0, s>>>(ex.d_plan, skip);
    CUDA_TRY(cudaGetLastError());
  }
  const int row_grid = (int)std::max<int64_t>(1, std::min<int64_t>((ex.lz_rows + 7) / 8, (int64_t)sms * 4));
  {  // every matrix iterates at first; each step's last block then writes the next list
    Launch L("k_lz_compact", SMUON_WORK_BYTES, 12.0 * h.n_mats, s);
    k_lz_compact<<<1, 1024, 0, s>>>(ex.d_plan, -1, skip);
    CUDA_TRY(cudaGetLastError());
  }
  for (int j = 0; j < kLanczosSteps; ++j) {
    {  // only the first launch's bytes are known on the host (later ones skip stopped matrices)
      Launch L("k_lz_matvec", SMUON_WORK_BYTES, j == 0 ? ex.lz_matvec_bytes : 0.0, s);
      k_lz_matvec<<<row_grid, 256, 0, s>>>(ex.d_plan, j, skip);
      CUDA_TRY(cudaGetLastError());
    }
    Launch L("k_lz_step", SMUON_WORK_BYTES, 4.0 * ex.lz_rows * (4.0 * (j + 1) + 6.0), s);
    k_lz_step<<<mat_grid, 256, 0, s>>>(ex.d_plan, j, skip);
    CUDA_TRY(cudaGetLastError());
  }
  Launch L("k_lz_finish", SMUON_WORK_BYTES, 8.0 * kLanczosSteps * h.n_mats, s);
  k_lz_finish<<<(h.n_mats * 32 + 255) / 256, 256, 0, s>>>(ex.d_plan, skip);  // one warp per matrix
  CUDA_TRY(cudaGetLastError());
  return SMUON_OK;
}

smuon_status run_ns(const NsExec& ex, const int32_t* skip, cudaStream_t s) {
  const PlanHeader& h = ex.h;
  const DevInfo& di = ex.di;
  smuon_status st;
  {
    const int grid = std::min(h.total_mom_tiles, di.sms * 8);
    {
      Launch L("k_momentum", SMUON_WORK_BYTES, ex.mom_bytes, s);
      k_momentum<<<std::max(grid, 1), 256, 0, s>>>(ex.d_plan, skip);
      CUDA_TRY(cudaGetLastError());
    }
    Launch L("k_norm_finalize", SMUON_WORK_BYTES, 4.0 * kMomSlots * h.total_mom_tiles, s);
    k_norm_finalize<<<std::max(h.n_mats, 1), 256, 0, s>>>(ex.d_plan, skip);
    CUDA_TRY(cudaGetLastError());
  }
  const bool emit_q = (ex.flags & SMUON_NS_EMIT_Q) != 0;
  if (ex.flags & SMUON_NS_GRAM_ONLY) {
    // A_0 = X_0 X_0^T; per step B_k = bA_k + cA_k^2 (Q_1 = aI + B_0 from its epilogue),
    // Q_{k+1} = aQ_k + B_k Q_k, and A_{k+1} = P_k (P_k A_k) except after the last step; then
    // U = s Q_K X_0 from the f32-accumulated Q_K in the workspace (split operands in split mode)
    auto run = [&](int stg, int k) {
      return launch_gemm(ex.d_plan, h, stg, k, skip, di, s, ex.sflops[stg], ex.sissued[stg]);
    };
    if ((st = run(ST_GRAM, 0)) != SMUON_OK) return st;
    for (int k = 0; k < ex.iters; ++k) {
      if ((st = run(ST_POLY, k)) != SMUON_OK) return st;
      if (k >= 1 && (st = run(ST_QAXPY, k)) != SMUON_OK) return st;
      if (k + 1 < ex.iters) {
        if ((st = run(ST_AA1, k)) != SMUON_OK) return st;
        if ((st = run(ST_AA2, k)) != SMUON_OK) return st;
      }
    }
    return run(ST_QX, ex.iters);
  }
  auto issued = [&](int stg, int k) { return k < 8 ? ex.sissued_lead[k][stg] : ex.sissued[stg]; };
  for (int k = 0; k < ex.iters; ++k) {
    if ((st = launch_gemm(ex.d_plan, h, ST_GRAM, k, skip, di, s, ex.sflops[ST_GRAM], issued(ST_GRAM, k))) != SMUON_OK) return st;
    if (k == 0 && (ex.flags & SMUON_NS_SPECTRAL) && (st = run_lanczos(ex, skip, s)) != SMUON_OK) return st;
    if (ex.c != 0.f && (st = launch_gemm(ex.d_plan, h, ST_POLY, k, skip, di, s, ex.sflops[ST_POLY], issued(ST_POLY, k))) != SMUON_OK)
      return st;
    if ((st = launch_gemm(ex.d_plan, h, ST_AXPY, k, skip, di, s, ex.sflops[ST_AXPY], issued(ST_AXPY, k))) != SMUON_OK) return st;
    if (emit_q && k >= 1 &&
        (st = launch_gemm(ex.d_plan, h, ST_QAXPY, k, skip, di, s, ex.sflops[ST_QAXPY], ex.sissued[ST_QAXPY])) != SMUON_OK)
      return st;
  }
  return SMUON_OK;
}

smuon_status enqueue_ns(const NsRequest& rq, void* ws, size_t ws_bytes, int32_t* d_status, const int32_t* skip,
                        cudaStream_t s) {
  NsExec ex;
  smuon_status st = prepare_ns(rq, ws, ws_bytes, d_status, s, &ex);
  if (st != SMUON_OK) return st;
  return run_ns(ex, skip, s);
}

// ------------------------------------------------------------------ elementwise tables
struct EwBuild {
  std::vector<EwLayer> layers;
  std::vector<std::vector<EwSrc>> srcs;  // per layer
};

bool vec_ok(const void* p, int64_t ld, int32_t cols, int esz) {
  return ld == cols && (reinterpret_cast<uintptr_t>(p) % 16 == 0) && esz > 0;
}

int ew_grid(int64_t chunks, const DevInfo& di) {
  const int64_t want = (chunks + 255) / 256;
  return (int)std::max<int64_t>(1, std::min<int64_t>(want, (int64_t)di.sms * 16));
}

// splits layers into launches of at most kEwMaxLayers layers / kEwMaxSrcs sources
template <class F>
smuon_status for_each_ew_launch(const EwBuild& eb, const EwTable& proto, F&& launch) {
  std::unique_ptr<EwTable> holder(new EwTable());  // large parameter block, launched by value
  EwTable& tb = *holder;
  size_t i = 0;
  while (i < eb.layers.size()) {
    tb = proto;
    tb.n_layers = 0;
    int nsrc = 0;
    int64_t chunks = 0;
    tb.any_packed = 0;
    while (i < eb.layers.size() && tb.n_layers < kEwMaxLayers &&
           nsrc + (int)eb.srcs[i].size() <= kEwMaxSrcs) {
      EwLayer L = eb.layers[i];
      L.chunk_begin = chunks;
      L.src_first = nsrc;
      for (const EwSrc& e : eb.srcs[i]) tb.srcs[nsrc++] = e;
      chunks += 16 * ((L.n + 127) / 128);
      if (L.packed_out) tb.any_packed = 1;
      tb.layers[tb.n_layers++] = L;
      ++i;
    }
    if (tb.n_layers == 0) return fail(SMUON_ERR_UNSUPPORTED, "a layer needs more than %d sources", kEwMaxSrcs);
    tb.total_chunks = chunks;
    smuon_status st = launch(tb);
    if (st != SMUON_OK) return st;
  }
  return SMUON_OK;
}

}  // namespace

// ======================================================================== ABI
extern "C" {

const char* smuon_last_error(void) { return g_err.c_str(); }

int64_t smuon_launch_count(void) { return g_launches.load(); }

void smuon_trace_enable(int32_t on) {
  std::lock_guard<std::mutex> lk(g_tr_mu);
  g_tr_on = on != 0;
}

int32_t smuon_trace_read(smuon_trace_rec* out, int32_t max_recs) {
  std::vector<TraceRec> recs;
  {
    std::lock_guard<std::mutex> lk(g_tr_mu);
    if (!out) return (int32_t)g_tr.size();
    recs.swap(g_tr);
  }
  int32_t n = 0;
  for (const TraceRec& r : recs) {
    float ms = -1.f;
    if (cudaEventSynchronize(r.b) == cudaSuccess) cudaEventElapsedTime(&ms, r.a, r.b);
    if (out && n < max_recs) {
      smuon_trace_rec& o = out[n];
      memset(&o, 0, sizeof(o));
      strncpy(o.name, r.name, sizeof(o.name) - 1);
      o.kind = r.kind;
      o.work = r.work;
      o.nominal = r.nominal;
      o.ms = ms;
    }
    ++n;
  }
  std::lock_guard<std::mutex> lk(g_tr_mu);
  for (const TraceRec& r : recs) g_ev_free.emplace_back(r.a, r.b);
  return std::min(n, max_recs);
}
int32_t smuon_version(void) { return (1 << 16) | 0; }

smuon_status smuon_ns_workspace_bytes(const smuon_mat* M_in, int32_t n_mats, int32_t iters, uint32_t flags,
                                      size_t* bytes) {
  if (!bytes || !M_in) return fail(SMUON_ERR_INVALID_ARG, "NULL argument");
  if (n_mats < 1 || n_mats > 4096 || iters < 1 || iters > 64) return fail(SMUON_ERR_INVALID_ARG, "bad n_mats/iters");
  std::vector<smuon_mat> fake(M_in, M_in + n_mats);
  NsRequest rq{};
  rq.M_in = fake.data(); rq.U_out = fake.data(); rq.n_mats = n_mats; rq.iters = iters; rq.flags = flags;
  rq.c = 1.f;  // size for the quintic case (the cubic needs less)
  std::vector<smuon_mat> q(n_mats);
  rq.Q_out = (flags & SMUON_NS_EMIT_Q) ? q.data() : nullptr;
  Builder B;
  smuon_status st = build_plan(rq, nullptr, &B);
  if (st != SMUON_OK) return st;
  *bytes = B.L.total;
  return SMUON_OK;
}

smuon_status smuon_ns(const smuon_mat* M_in, const smuon_mat* U_out, int32_t n_mats, const smuon_mat* G,
                      float beta, float a, float b, float c, int32_t iters, float eps, uint32_t flags,
                      const smuon_mat* Q_out, const int32_t* d_skip_if, void* ws, size_t ws_bytes,
                      int32_t* d_status, void* stream) {
  NsRequest rq{};
  rq.M_in = M_in; rq.U_out = U_out; rq.n_mats = n_mats; rq.G = G; rq.beta = beta;
  rq.a = a; rq.b = b; rq.c = c; rq.iters = iters; rq.eps = eps; rq.flags = flags; rq.Q_out = Q_out;
  smuon_status st = validate_ns(rq);
  if (st != SMUON_OK) return st;
  return enqueue_ns(rq, ws, ws_bytes, d_status, d_skip_if, reinterpret_cast<cudaStream_t>(stream));
}

smuon_status smuon_sign_pack(const smuon_mat* U, int32_t M, uint32_t* packed, int8_t* signs_i8, void* stream) {
  if (!U) return fail(SMUON_ERR_INVALID_ARG, "U is NULL");
  if (M < 1 || M > kMaxWorkers) return fail(SMUON_ERR_UNSUPPORTED, "M=%d must be in 1..%d", M, kMaxWorkers);
  if (!packed && !signs_i8) return fail(SMUON_ERR_INVALID_ARG, "give packed and/or signs_i8");
  for (int k = 0; k < M; ++k) {
    smuon_status st = check_mat(U[k], "U", k, true, true, true);  // I8: sign matrices (entry >= 0 -> +1)
    if (st != SMUON_OK) return st;
    if (!same_shape(U[k], U[0]) || U[k].dtype != U[0].dtype)
      return fail(SMUON_ERR_SHAPE, "U[%d] differs from U[0] in shape or dtype", k);
  }
  DevInfo di;
  smuon_status st = device_info(&di);
  if (st != SMUON_OK) return st;
  EwBuild eb;
  EwLayer L{};
  L.rows = U[0].rows; L.cols = U[0].cols; L.n = (int64_t)L.rows * L.cols;
  L.words = 4 * ((L.n + 127) / 128);
  L.vec = 1;
  std::vector<EwSrc> srcs;
  for (int k = 0; k < M; ++k) {
    srcs.push_back(EwSrc{U[k].data, U[k].ld});
    if (!vec_ok(U[k].data, U[k].ld, U[k].cols, 1)) L.vec = 0;
  }
  eb.layers.push_back(L);
  eb.srcs.push_back(srcs);
  EwTable proto{};
  proto.M = M; proto.src_dtype = U[0].dtype;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  return for_each_ew_launch(eb, proto, [&](const EwTable& tb) -> smuon_status {
    const double n = (double)tb.layers[0].n;
    Launch L("k_sign_pack", SMUON_WORK_BYTES,
             n * M * dtype_size(U[0].dtype) + (packed ? n * M / 8.0 : 0.0) + (signs_i8 ? n * M : 0.0), s);
    k_sign_pack<<<ew_grid(tb.total_chunks, di), 256, 0, s>>>(tb, packed, signs_i8);
    CUDA_TRY(cudaGetLastError());
    return SMUON_OK;
  });
}

smuon_status smuon_vote(const uint32_t* packed, const int8_t* signs_i8, int32_t M, int64_t N, int8_t tie_value,
                        int8_t* vote, void* stream) {
  if ((packed == nullptr) == (signs_i8 == nullptr))
    return fail(SMUON_ERR_INVALID_ARG, "give exactly one of packed and signs_i8");
  if (!vote) return fail(SMUON_ERR_INVALID_ARG, "vote is NULL");
  if (M < 1 || M > kMaxWorkers) return fail(SMUON_ERR_UNSUPPORTED, "M=%d must be in 1..%d", M, kMaxWorkers);
  if (N < 1) return fail(SMUON_ERR_SHAPE, "N=%lld must be positive", (long long)N);
  if (tie_value < -1 || tie_value > 1) return fail(SMUON_ERR_INVALID_ARG, "tie_value must be -1, 0 or 1");
  if (packed && reinterpret_cast<uintptr_t>(packed) % 16) return fail(SMUON_ERR_INVALID_ARG, "packed must be 16-byte aligned");
  DevInfo di;
  smuon_status st = device_info(&di);
  if (st != SMUON_OK) return st;
  const int64_t nw = (N + 31) / 32;
  const int grid = (int)std::max<int64_t>(1, std::min<int64_t>((nw + 255) / 256, (int64_t)di.sms * 16));
  Launch L("k_vote", SMUON_WORK_BYTES, (double)N * (packed ? M / 8.0 : (double)M) + (double)N,
           reinterpret_cast<cudaStream_t>(stream));
  k_vote<<<grid, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(packed, signs_i8, M, N, 4 * ((N + 127) / 128),
                                                                    tie_value, vote);
  CUDA_TRY(cudaGetLastError());
  return SMUON_OK;
}

}  // extern "C"

namespace {

struct UpdExec {
  std::vector<EwTable> tables;   // one per launch
  std::vector<double> bytes;
  int source = 0;                // 0 = U (fused vote), 1 = votes / dense
  uint32_t vote_kind = 0;
  DevInfo di;
};

smuon_status prepare_update(const smuon_mat* W, int32_t n_layers, const smuon_mat* U, const smuon_mat* votes,
                            const smuon_mat* dense, int32_t M, float eta, int8_t tie_value, uint32_t vote_kind,
                            uint32_t* const* packed_out, int8_t* const* vote_out, int32_t* d_status,
                            UpdExec* ex) {
  if (n_layers < 1) return fail(SMUON_ERR_INVALID_ARG, "n_layers < 1");
  const int nsrc = (U != nullptr) + (votes != nullptr) + (dense != nullptr);
  if (nsrc != 1) return fail(SMUON_ERR_INVALID_ARG, "exactly one of U, votes, dense must be given");
  // W == NULL: signs, message and vote only (the local polar step's input, or an exchange's payload)
  if (!W && !(U && (packed_out || vote_out)))
    return fail(SMUON_ERR_INVALID_ARG, "W may be NULL only with the U source and packed_out or vote_out");
  if (U && (M < 1 || M > kMaxWorkers)) return fail(SMUON_ERR_UNSUPPORTED, "M=%d must be in 1..%d", M, kMaxWorkers);
  if (tie_value < -1 || tie_value > 1) return fail(SMUON_ERR_INVALID_ARG, "tie_value must be -1, 0 or 1");
  const bool test_starve = (vote_kind & SMUON_VOTE_TEST_WAIT_EXPIRY) != 0;
  vote_kind &= ~SMUON_VOTE_TEST_WAIT_EXPIRY;
  if (vote_kind > SMUON_VOTE_INT8) return fail(SMUON_ERR_INVALID_ARG, "unknown vote_kind %u", vote_kind);
  if (!U && (packed_out || vote_out)) return fail(SMUON_ERR_INVALID_ARG, "packed_out/vote_out need the U source");
  int32_t src_dtype = -1;
  EwBuild eb;
  for (int l = 0; l < n_layers; ++l) {
    smuon_status st = SMUON_OK;
    const smuon_mat& shape = W ? W[l] : U[(int64_t)l * M];  // layer shape (the first worker's U without W)
    if (W && (st = check_mat(W[l], "W", l, true, true, false)) != SMUON_OK) return st;
    EwLayer L{};
    if (W) { L.w = W[l].data; L.w_ld = W[l].ld; L.w_dtype = W[l].dtype; }
    L.rows = shape.rows; L.cols = shape.cols; L.n = (int64_t)L.rows * L.cols;
    L.words = 4 * ((L.n + 127) / 128);
    L.vec = W ? vec_ok(W[l].data, W[l].ld, W[l].cols, 1) : 1;
    std::vector<EwSrc> srcs;
    if (U) {
      for (int k = 0; k < M; ++k) {
        const smuon_mat& u = U[(int64_t)l * M + k];
        if ((st = check_mat(u, "U", l * M + k, true, true, true, true)) != SMUON_OK) return st;
        if (!same_shape(u, shape)) return fail(SMUON_ERR_SHAPE, "U[%d] shape differs from W[%d]", l * M + k, l);
        if (src_dtype >= 0 && u.dtype != src_dtype) return fail(SMUON_ERR_DTYPE, "all U must share one dtype");
        src_dtype = u.dtype;
        // a 1-bit message is read word by word (16-byte aligned, checked above); W decides the fast path
        if (u.dtype != SMUON_BITS && !vec_ok(u.data, u.ld, u.cols, 1)) L.vec = 0;
        srcs.push_back(EwSrc{u.data, u.ld});
      }
      if (packed_out && packed_out[l]) {
        if (src_dtype == SMUON_BITS)
          return fail(SMUON_ERR_INVALID_ARG, "packed_out with 1-bit message sources: they are the message");
        if (src_dtype == SMUON_I8)
          return fail(SMUON_ERR_UNSUPPORTED, "packed_out needs F32 or BF16 U (pack I8 signs with smuon_sign_pack)");
        if (reinterpret_cast<uintptr_t>(packed_out[l]) % 16)
          return fail(SMUON_ERR_INVALID_ARG, "packed_out[%d] must be 16-byte aligned", l);
        L.packed_out = packed_out[l];
      }
      if (vote_out) L.vote_out = vote_out[l];
    } else {
      const smuon_mat& d = votes ? votes[l] : dense[l];
      if ((st = check_mat(d, votes ? "votes" : "dense", l, !votes, !votes, votes != nullptr)) != SMUON_OK) return st;
      if (!same_shape(d, W[l])) return fail(SMUON_ERR_SHAPE, "source %d shape differs from W", l);
      if (src_dtype >= 0 && d.dtype != src_dtype) return fail(SMUON_ERR_DTYPE, "all sources must share one dtype");
      src_dtype = d.dtype;
      if (!vec_ok(d.data, d.ld, d.cols, 1)) L.vec = 0;
      srcs.push_back(EwSrc{d.data, d.ld});
    }
    eb.layers.push_back(L);
    eb.srcs.push_back(srcs);
  }
  smuon_status st = device_info(&ex->di);
  if (st != SMUON_OK) return st;
  EwTable proto{};
  proto.M = U ? M : 1;
  proto.tie = tie_value;
  proto.src_dtype = src_dtype;
  proto.eta = eta;
  proto.test_starve = test_starve ? 1 : 0;
  proto.status = d_status;
  ex->source = U ? 0 : 1;
  ex->vote_kind = vote_kind;
  ex->tables.clear();
  ex->bytes.clear();
  return for_each_ew_launch(eb, proto, [&](const EwTable& tb) -> smuon_status {
    double bytes = 0;
    for (int l = 0; l < tb.n_layers; ++l) {
      const EwLayer& Ly = tb.layers[l];
      const double src_bytes = src_dtype == SMUON_BITS ? tb.M / 8.0 : (double)tb.M * dtype_size(src_dtype);
      bytes += (double)Ly.n * (src_bytes + (Ly.w ? 2 * dtype_size(Ly.w_dtype) : 0));
      if (Ly.packed_out) bytes += (double)Ly.n * tb.M / 8.0;
      if (Ly.vote_out) bytes += (double)Ly.n;
    }
    ex->tables.push_back(tb);
    ex->bytes.push_back(bytes);
    return SMUON_OK;
  });
}

smuon_status run_update(const UpdExec& ex, cudaStream_t s) {
  for (size_t i = 0; i < ex.tables.size(); ++i) {
    const EwTable& tb = ex.tables[i];
    const int grid = ew_grid(tb.total_chunks, ex.di);
    if (ex.source == 0) {
      Launch L(tb.src_dtype == SMUON_BITS ? (bits_tma_eligible(tb) ? "k_vote_update_bits_tma" : "k_vote_update_bits")
               : ex.vote_kind == SMUON_VOTE_POPCOUNT ? "k_vote_update_popcount" : "k_vote_update_int8",
               SMUON_WORK_BYTES, ex.bytes[i], s);
      CUDA_TRY(launch_vote_update(tb, ex.vote_kind == SMUON_VOTE_POPCOUNT, grid, ex.di.sms, s));
    } else {
      Launch L("k_update_src", SMUON_WORK_BYTES, ex.bytes[i], s);
      k_update_src<<<grid, 256, 0, s>>>(tb);
    }
    CUDA_TRY(cudaGetLastError());
  }
  return SMUON_OK;
}

}  // namespace

// plan handles: host objects holding everything needed to relaunch a call
struct smuon_plan_s {
  int kind;  // 0 = Newton-Schulz, 1 = update
  NsExec ns;
  UpdExec upd;
};

extern "C" {

smuon_status smuon_update(const smuon_mat* W, int32_t n_layers, const smuon_mat* U, const smuon_mat* votes,
                          const smuon_mat* dense, int32_t M, float eta, int8_t tie_value, uint32_t vote_kind,
                          uint32_t* const* packed_out, int8_t* const* vote_out, int32_t* d_status, void* stream) {
  UpdExec ex;
  smuon_status st =
      prepare_update(W, n_layers, U, votes, dense, M, eta, tie_value, vote_kind, packed_out, vote_out, d_status, &ex);
  if (st != SMUON_OK) return st;
  return run_update(ex, reinterpret_cast<cudaStream_t>(stream));
}

smuon_status smuon_ns_plan_create(const smuon_mat* M_in, const smuon_mat* U_out, int32_t n_mats, const smuon_mat* G,
                                  float beta, float a, float b, float c, int32_t iters, float eps, uint32_t flags,
                                  const smuon_mat* Q_out, void* ws, size_t ws_bytes, int32_t* d_status, void* stream,
                                  smuon_plan* out) {
  if (!out) return fail(SMUON_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  NsRequest rq{};
  rq.M_in = M_in; rq.U_out = U_out; rq.n_mats = n_mats; rq.G = G; rq.beta = beta;
  rq.a = a; rq.b = b; rq.c = c; rq.iters = iters; rq.eps = eps; rq.flags = flags; rq.Q_out = Q_out;
  smuon_status st = validate_ns(rq);
  if (st != SMUON_OK) return st;
  smuon_plan_s* p = new smuon_plan_s();
  p->kind = 0;
  st = prepare_ns(rq, ws, ws_bytes, d_status, reinterpret_cast<cudaStream_t>(stream), &p->ns);
  if (st != SMUON_OK) {
    delete p;
    return st;
  }
  *out = p;
  return SMUON_OK;
}

smuon_status smuon_ns_execute(smuon_plan plan, const int32_t* d_skip_if, void* stream) {
  if (!plan || plan->kind != 0) return fail(SMUON_ERR_INVALID_ARG, "not a Newton-Schulz plan");
  return run_ns(plan->ns, d_skip_if, reinterpret_cast<cudaStream_t>(stream));
}

smuon_status smuon_update_plan_create(const smuon_mat* W, int32_t n_layers, const smuon_mat* U,
                                      const smuon_mat* votes, const smuon_mat* dense, int32_t M, float eta,
                                      int8_t tie_value, uint32_t vote_kind, uint32_t* const* packed_out,
                                      int8_t* const* vote_out, int32_t* d_status, smuon_plan* out) {
  if (!out) return fail(SMUON_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  smuon_plan_s* p = new smuon_plan_s();
  p->kind = 1;
  smuon_status st = prepare_update(W, n_layers, U, votes, dense, M, eta, tie_value, vote_kind, packed_out,
                                   vote_out, d_status, &p->upd);
  if (st != SMUON_OK) {
    delete p;
    return st;
  }
  *out = p;
  return SMUON_OK;
}

smuon_status smuon_update_execute(smuon_plan plan, void* stream) {
  if (!plan || plan->kind != 1) return fail(SMUON_ERR_INVALID_ARG, "not an update plan");
  return run_update(plan->upd, reinterpret_cast<cudaStream_t>(stream));
}

void smuon_plan_destroy(smuon_plan plan) { delete plan; }

smuon_status cachemuon_workspace_bytes(const smuon_mat* M_t, size_t* bytes) {
  if (!M_t || !bytes) return fail(SMUON_ERR_INVALID_ARG, "NULL argument");
  NsRequest rq{};
  rq.M_in = M_t; rq.U_out = M_t; rq.n_mats = 1; rq.iters = 1; rq.probe = true; rq.Q_out = M_t;
  Builder B;
  smuon_status st = build_plan(rq, nullptr, &B);
  if (st != SMUON_OK) return st;
  *bytes = B.L.total;
  return SMUON_OK;
}

smuon_status cachemuon_reuse_probe(const smuon_mat* Q, const smuon_mat* M_t, const smuon_mat* D_hat, float gamma,
                                   float eps, float* d_err, int32_t* d_accept, cachemuon_counters* d_counters,
                                   void* ws, size_t ws_bytes, int32_t* d_status, void* stream) {
  if (!M_t || !D_hat || !d_err || !d_accept) return fail(SMUON_ERR_INVALID_ARG, "M_t, D_hat, d_err, d_accept must not be NULL");
  smuon_status st;
  if ((st = check_mat(*M_t, "M_t", 0, true, false, false)) != SMUON_OK) return st;
  if ((st = check_mat(*D_hat, "D_hat", 0, true, true, false)) != SMUON_OK) return st;
  if (!same_shape(*M_t, *D_hat)) return fail(SMUON_ERR_SHAPE, "D_hat shape differs from M_t");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  DevInfo di;
  if ((st = device_info(&di)) != SMUON_OK) return st;
  if (!Q) {
    Launch L("k_probe_nocache", SMUON_WORK_BYTES, 8.0, s);
    k_probe_nocache<<<1, 1, 0, s>>>(d_err, d_accept, d_counters);
    CUDA_TRY(cudaGetLastError());
    return SMUON_OK;
  }
  const int m = std::min(M_t->rows, M_t->cols);
  if ((st = check_mat(*Q, "Q", 0, false, true, false)) != SMUON_OK) return st;
  if (Q->rows != m || Q->cols != m) return fail(SMUON_ERR_SHAPE, "Q must be %dx%d", m, m);
  if (reinterpret_cast<uintptr_t>(Q->data) % 16 || (Q->ld * 2) % 16)
    return fail(SMUON_ERR_INVALID_ARG, "Q must be 16-byte aligned with ld a multiple of 8 (TMA operand)");
  NsRequest rq{};
  rq.M_in = M_t; rq.U_out = D_hat; rq.n_mats = 1; rq.iters = 1; rq.eps = eps; rq.flags = 0;
  rq.Q_out = Q; rq.probe = true; rq.gamma = gamma;
  Builder B;
  if ((st = build_plan(rq, nullptr, &B)) != SMUON_OK) return st;
  if ((st = check_ws(ws, ws_bytes, B.L.total)) != SMUON_OK) return st;
  if ((st = build_plan(rq, reinterpret_cast<char*>(ws), &B)) != SMUON_OK) return st;
  B.h.status = d_status;
  B.h.d_err = d_err;
  B.h.d_accept = d_accept;
  B.h.counters = d_counters;
  if ((st = upload_plan(B, s)) != SMUON_OK) return st;
  const Plan* d_plan = reinterpret_cast<const Plan*>(ws);
  {
    Launch L("k_momentum", SMUON_WORK_BYTES, momentum_bytes(rq, B.h), s);
    k_momentum<<<std::max(1, std::min(B.h.total_mom_tiles, di.sms * 8)), 256, 0, s>>>(d_plan, nullptr);
    CUDA_TRY(cudaGetLastError());
  }
  {
    Launch L("k_norm_finalize", SMUON_WORK_BYTES, 4.0 * kMomSlots * B.h.total_mom_tiles, s);
    k_norm_finalize<<<std::max(B.h.n_mats, 1), 256, 0, s>>>(d_plan, nullptr);
    CUDA_TRY(cudaGetLastError());
  }
  if ((st = launch_gemm(d_plan, B.h, ST_REUSE, 0, nullptr, di, s, stage_flops(B, ST_REUSE),
                        stage_issued(B, ST_REUSE))) != SMUON_OK)
    return st;
  if ((st = launch_gemm(d_plan, B.h, ST_PROBE, 0, nullptr, di, s, stage_flops(B, ST_PROBE),
                        stage_issued(B, ST_PROBE))) != SMUON_OK)
    return st;
  Launch L("k_probe_finalize", SMUON_WORK_BYTES, 16.0 * B.h.total_tiles[ST_PROBE], s);
  k_probe_finalize<<<1, 32, 0, s>>>(d_plan);
  CUDA_TRY(cudaGetLastError());
  return SMUON_OK;
}

// LionMuon workspace: the mean buffers and directions of a Muon step, then the NS workspace
// LionMuon Muon-step workspace. Mean reading: per layer the f32 mean of G_hat
// and the f32 direction, then the Newton-Schulz workspace of n_layers
// problems. Vote reading (SMUON_LION_MUON_VOTE): per layer the M workers' f32
// G_hat back to back (worker k at k * rows * cols), per (layer, worker) a bf16
// polar factor, then the workspace of n_layers * M problems. `means` and
// `dirs` are the Newton-Schulz inputs and outputs (worker-minor in the vote reading).
static smuon_status lion_layout(const lionmuon_state* st, int32_t iters, uint32_t ns_flags, size_t* mean_off,
                                size_t* dir_off, size_t* ns_off, size_t* total, std::vector<smuon_mat>* means,
                                std::vector<smuon_mat>* dirs, char* base) {
  const bool vote = (ns_flags & SMUON_LION_MUON_VOTE) != 0;
  const int per = vote ? st->workers : 1;
  size_t cur = 0;
  means->clear();
  dirs->clear();
  *mean_off = 0;
  for (int l = 0; l < st->n_layers; ++l) {
    const smuon_mat& w = st->W[l];
    for (int k = 0; k < per; ++k) {
      smuon_mat m{};
      m.rows = w.rows; m.cols = w.cols; m.ld = w.cols; m.dtype = SMUON_F32;
      m.data = base ? base + cur : nullptr;
      cur += (size_t)w.rows * w.cols * 4;
      means->push_back(m);
    }
    cur = (size_t)round_up((int64_t)cur, 256);
  }
  *dir_off = cur;
  for (int l = 0; l < st->n_layers; ++l) {
    const smuon_mat& w = st->W[l];
    for (int k = 0; k < per; ++k) {
      smuon_mat d{};
      d.rows = w.rows; d.cols = w.cols; d.ld = w.cols; d.dtype = vote ? SMUON_BF16 : SMUON_F32;
      d.data = base ? base + cur : nullptr;
      cur = (size_t)round_up((int64_t)(cur + (size_t)w.rows * w.cols * dtype_size(d.dtype)), 256);
      dirs->push_back(d);
    }
  }
  *ns_off = cur;
  size_t ns_bytes = 0;
  smuon_status s = smuon_ns_workspace_bytes(means->data(), (int32_t)means->size(), iters,
                                            ns_flags & ~SMUON_LION_MUON_VOTE, &ns_bytes);
  if (s != SMUON_OK) return s;
  *total = cur + ns_bytes;
  return SMUON_OK;
}

smuon_status lionmuon_workspace_bytes(const lionmuon_state* st, int32_t iters, uint32_t ns_flags, size_t* bytes) {
  if (!st || !bytes || !st->W || st->n_layers < 1) return fail(SMUON_ERR_INVALID_ARG, "bad state");
  size_t a, b, c, total;
  std::vector<smuon_mat> means, dirs;
  smuon_status s = lion_layout(st, iters, ns_flags, &a, &b, &c, &total, &means, &dirs, nullptr);
  if (s != SMUON_OK) return s;
  *bytes = total;
  return SMUON_OK;
}

smuon_status smuon_harness_gaussian(const smuon_mat* G, int32_t n_layers, int32_t workers,
                                    const smuon_grad_stream* gs, uint32_t step, void* stream) {
  if (!G || !gs) return fail(SMUON_ERR_INVALID_ARG, "G and gs must not be NULL");
  if (n_layers < 1 || workers < 1) return fail(SMUON_ERR_INVALID_ARG, "n_layers and workers must be >= 1");
  if ((int64_t)n_layers * workers > (1 << 20)) return fail(SMUON_ERR_INVALID_ARG, "too many matrices");
  smuon_status s;
  EwBuild eb;
  for (int l = 0; l < n_layers; ++l)
    for (int k = 0; k < workers; ++k) {
      const int i = l * workers + k;
      const smuon_mat& g = G[i];
      if ((s = check_mat(g, "G", i, true, false, false)) != SMUON_OK) return s;
      EwLayer L{};
      L.w = g.data; L.w_ld = g.ld; L.w_dtype = SMUON_F32;
      L.rows = g.rows; L.cols = g.cols; L.n = (int64_t)g.rows * g.cols;
      L.vec = vec_ok(g.data, g.ld, g.cols, 1);
      L.key0 = gs->seed_base + (uint32_t)k;
      L.key1 = gs->matrix_base + (uint32_t)l;
      eb.layers.push_back(L);
      eb.srcs.push_back({});
    }
  DevInfo di;
  if ((s = device_info(&di)) != SMUON_OK) return s;
  cudaStream_t strm = reinterpret_cast<cudaStream_t>(stream);
  EwTable proto{};
  proto.gen_step = step;
  proto.gen_sigma = gs->sigma;
  return for_each_ew_launch(eb, proto, [&](const EwTable& tb) -> smuon_status {
    double n = 0;
    for (int l = 0; l < tb.n_layers; ++l) n += 4.0 * (double)tb.layers[l].n;
    Launch L("k_harness_gaussian", SMUON_WORK_BYTES, n, strm);
    k_harness_gaussian<<<ew_grid(tb.total_chunks, di), 256, 0, strm>>>(tb);
    CUDA_TRY(cudaGetLastError());
    return SMUON_OK;
  });
}

smuon_status lionmuon_step(lionmuon_state* st, int32_t P, float beta1, float beta2, float eta, float a, float b,
                           float c, int32_t iters, int8_t tie_value, uint32_t ns_flags, const smuon_mat* G, void* ws,
                           size_t ws_bytes, int32_t* d_status, void* stream) {
  if (!st || !st->W || !st->mom) return fail(SMUON_ERR_INVALID_ARG, "state, W and mom must not be NULL");
  if (!G && !st->grad) return fail(SMUON_ERR_INVALID_ARG, "G is NULL and the state has no gradient stream");
  const bool gen = (G == nullptr);
  if (st->n_layers < 1) return fail(SMUON_ERR_INVALID_ARG, "n_layers < 1");
  const int M = st->workers;
  if (M < 1 || M > kMaxWorkers) return fail(SMUON_ERR_UNSUPPORTED, "workers=%d must be in 1..%d", M, kMaxWorkers);
  if (P < 0) return fail(SMUON_ERR_INVALID_ARG, "P must be >= 0 (0 = never a Muon step)");
  if (tie_value < -1 || tie_value > 1) return fail(SMUON_ERR_INVALID_ARG, "tie_value must be -1, 0 or 1");
  if (iters < 1 || iters > 64) return fail(SMUON_ERR_INVALID_ARG, "iters must be in 1..64");
  if (ns_flags & SMUON_NS_EMIT_Q) return fail(SMUON_ERR_INVALID_ARG, "ns_flags may not ask for SMUON_NS_EMIT_Q");
  if ((ns_flags & SMUON_LION_MUON_VOTE) && (int64_t)st->n_layers * M > 4096)
    return fail(SMUON_ERR_UNSUPPORTED, "the vote reading orthogonalises n_layers * workers <= 4096 matrices");
  smuon_status s;
  EwBuild eb;
  for (int l = 0; l < st->n_layers; ++l) {
    if ((s = check_mat(st->W[l], "W", l, true, true, false)) != SMUON_OK) return s;
    EwLayer L{};
    L.w = st->W[l].data; L.w_ld = st->W[l].ld; L.w_dtype = st->W[l].dtype;
    L.rows = st->W[l].rows; L.cols = st->W[l].cols; L.n = (int64_t)L.rows * L.cols;
    L.vec = vec_ok(L.w, L.w_ld, L.cols, 1);
    std::vector<EwSrc> srcs;
    if (gen) L.key1 = st->grad->matrix_base + (uint32_t)l;
    for (int k = 0; k < M; ++k) {
      const smuon_mat& mo = st->mom[(int64_t)l * M + k];
      if ((s = check_mat(mo, "mom", l * M + k, true, false, false)) != SMUON_OK) return s;
      if (!same_shape(mo, st->W[l])) return fail(SMUON_ERR_SHAPE, "mom of layer %d differs from W's shape", l);
      if (!vec_ok(mo.data, mo.ld, mo.cols, 1)) L.vec = 0;
      srcs.push_back(EwSrc{mo.data, mo.ld});
      if (gen) {
        srcs.push_back(EwSrc{nullptr, 0});  // drawn in-kernel
        continue;
      }
      const smuon_mat& g = G[(int64_t)l * M + k];
      if ((s = check_mat(g, "G", l * M + k, true, false, false)) != SMUON_OK) return s;
      if (!same_shape(g, st->W[l])) return fail(SMUON_ERR_SHAPE, "G of layer %d differs from W's shape", l);
      if (!vec_ok(g.data, g.ld, g.cols, 1)) L.vec = 0;
      srcs.push_back(EwSrc{g.data, g.ld});
    }
    eb.layers.push_back(L);
    eb.srcs.push_back(srcs);
  }
  DevInfo di;
  if ((s = device_info(&di)) != SMUON_OK) return s;
  cudaStream_t strm = reinterpret_cast<cudaStream_t>(stream);
  const int64_t t_next = st->t + 1;
  const bool muon = P > 0 && (t_next % P) == 0;
  EwTable proto{};
  proto.M = M; proto.tie = tie_value; proto.src_dtype = SMUON_F32; proto.eta = eta;
  proto.beta1 = beta1; proto.beta2 = beta2;
  proto.c1 = 1.f - beta1;  // float32 (1 - beta), as in the reading of the EMA
  proto.c2 = 1.f - beta2;
  if (gen) {
    proto.gen_on = 1;
    proto.gen_seed = st->grad->seed_base;
    proto.gen_step = (uint32_t)t_next;
    proto.gen_sigma = st->grad->sigma;
  }
  const double g_bytes = gen ? 0.0 : 4.0;  // gradient bytes read per entry and worker
  if (!muon) {
    s = for_each_ew_launch(eb, proto, [&](const EwTable& tb) -> smuon_status {
      double n = 0;
      for (int l = 0; l < tb.n_layers; ++l)
        n += (double)tb.layers[l].n * ((8.0 + g_bytes) * M + 2 * dtype_size(tb.layers[l].w_dtype));
      Launch L("k_lion_sign", SMUON_WORK_BYTES, n, strm);
      k_lion_sign<<<ew_grid(tb.total_chunks, di), 256, 0, strm>>>(tb);
      CUDA_TRY(cudaGetLastError());
      return SMUON_OK;
    });
    if (s != SMUON_OK) return s;
    st->t = t_next;
    return SMUON_OK;
  }
  size_t mean_off, dir_off, ns_off, total;
  std::vector<smuon_mat> means, dirs;
  if ((s = lion_layout(st, iters, ns_flags, &mean_off, &dir_off, &ns_off, &total, &means, &dirs, nullptr)) != SMUON_OK)
    return s;
  if ((s = check_ws(ws, ws_bytes, total)) != SMUON_OK) return s;
  char* base = reinterpret_cast<char*>(ws);
  if ((s = lion_layout(st, iters, ns_flags, &mean_off, &dir_off, &ns_off, &total, &means, &dirs, base)) != SMUON_OK)
    return s;
  const bool vote = (ns_flags & SMUON_LION_MUON_VOTE) != 0;
  for (int l = 0; l < st->n_layers; ++l) {
    eb.layers[l].aux = means[(size_t)l * (vote ? M : 1)].data;
    eb.layers[l].vec_aux = (eb.layers[l].vec != 0);
  }
  proto.ghat_out = vote ? 1 : 0;
  s = for_each_ew_launch(eb, proto, [&](const EwTable& tb) -> smuon_status {
    double n = 0;
    for (int l = 0; l < tb.n_layers; ++l) n += (double)tb.layers[l].n * ((8.0 + g_bytes) * M + (vote ? 4.0 * M : 4.0));
    Launch L("k_lion_mean", SMUON_WORK_BYTES, n, strm);
    k_lion_mean<<<ew_grid(tb.total_chunks, di), 256, 0, strm>>>(tb);
    CUDA_TRY(cudaGetLastError());
    return SMUON_OK;
  });
  if (s != SMUON_OK) return s;
  NsRequest rq{};
  rq.M_in = means.data(); rq.U_out = dirs.data(); rq.n_mats = (int32_t)means.size(); rq.iters = iters;
  rq.a = a; rq.b = b; rq.c = c; rq.eps = 1e-7f; rq.flags = ns_flags & ~SMUON_LION_MUON_VOTE;
  if ((s = validate_ns(rq)) != SMUON_OK) return s;
  if ((s = enqueue_ns(rq, base + ns_off, total - ns_off, d_status, nullptr, strm)) != SMUON_OK) return s;
  if (vote)  // Sign-Muon step on the orthogonalised G_hat: fused sign / popcount vote / update
    s = smuon_update(st->W, st->n_layers, dirs.data(), nullptr, nullptr, M, eta, tie_value, SMUON_VOTE_POPCOUNT,
                     nullptr, nullptr, d_status, stream);
  else
    s = smuon_update(st->W, st->n_layers, nullptr, nullptr, dirs.data(), 1, eta, 0, 0, nullptr, nullptr, d_status,
                     stream);
  if (s != SMUON_OK) return s;
  st->t = t_next;
  return SMUON_OK;
}

}  // extern "C"

// ======================================================================== no-allocation variant
// smuon_ns_static runs the same momentum + Newton-Schulz kernels as smuon_ns,
// but its scratch (plan, norm partials, operand buffers) lives in this
// file-scope device array instead of a caller-provided workspace. Every GPU
// that loads the library holds the array until the process exits.
static __device__ __align__(256) unsigned char g_ns_static_scratch[SMUON_NS_STATIC_SCRATCH_BYTES];

namespace {
std::mutex g_static_mu;
void* g_static_ptr[256] = {nullptr};
CUcontext g_static_ctx[256] = {nullptr};

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);

// the calling thread's current context (the device's primary context for runtime API callers)
CUcontext current_context() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  CUcontext c = nullptr;
  if (fn) fn(&c);
  return c;
}

// host code must not hand the symbol itself to a kernel: it is a host-side
// stand-in, so the device address is looked up once per device and context
// (a context created anew, e.g. after cudaDeviceReset, may load the module at
// another address, so a changed context handle looks it up again)
smuon_status static_scratch(void** out) {
  int dev = 0;
  CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 256) return fail(SMUON_ERR_UNSUPPORTED, "device index %d out of range", dev);
  const CUcontext ctx = current_context();  // null before the runtime has made one current on this thread
  std::lock_guard<std::mutex> lk(g_static_mu);
  if (!g_static_ptr[dev] || !ctx || g_static_ctx[dev] != ctx) {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_ns_static_scratch);  // initialises the context if needed
    if (e != cudaSuccess || !p)
      return fail(SMUON_ERR_CUDA, "cudaGetSymbolAddress of the static scratch failed: %s", cudaGetErrorString(e));
    g_static_ptr[dev] = p;
    g_static_ctx[dev] = current_context();
  }
  *out = g_static_ptr[dev];
  return SMUON_OK;
}
}  // namespace

extern "C" smuon_status smuon_ns_static(const smuon_mat* M_in, const smuon_mat* U_out, int32_t n_mats,
                                        const smuon_mat* G, float beta, float a, float b, float c, int32_t iters,
                                        float eps, uint32_t flags, const smuon_mat* Q_out, const int32_t* d_skip_if,
                                        int32_t* d_status, void* stream) {
  NsRequest rq{};
  rq.M_in = M_in; rq.U_out = U_out; rq.n_mats = n_mats; rq.G = G; rq.beta = beta;
  rq.a = a; rq.b = b; rq.c = c; rq.iters = iters; rq.eps = eps; rq.flags = flags; rq.Q_out = Q_out;
  smuon_status st = validate_ns(rq);
  if (st != SMUON_OK) return st;
  Builder B;
  if ((st = build_plan(rq, nullptr, &B)) != SMUON_OK) return st;
  if (B.L.total > (size_t)SMUON_NS_STATIC_SCRATCH_BYTES)
    return fail(SMUON_ERR_WORKSPACE,
                "this batch needs %zu bytes of scratch; smuon_ns_static holds at most %u bytes (use smuon_ns "
                "with a workspace)",
                B.L.total, (unsigned)SMUON_NS_STATIC_SCRATCH_BYTES);
  void* ws = nullptr;
  if ((st = static_scratch(&ws)) != SMUON_OK) return st;
  return enqueue_ns(rq, ws, SMUON_NS_STATIC_SCRATCH_BYTES, d_status, d_skip_if,
                    reinterpret_cast<cudaStream_t>(stream));
}
