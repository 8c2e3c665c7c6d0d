// pl_debug_gemm: a plain GEMM through the persistent tcgen05 kernel (test hook).
#include "../../include/pl_debug.h"
#include "gemm.h"

using namespace pl;

extern "C" pl_status pl_debug_gemm_out(const void* A, int a_mn, int64_t lda, const void* B, int b_mn,
                                       int64_t ldb, float* D, int64_t ldd, int out_path, int64_t M, int64_t N,
                                       int64_t K, uint32_t mode, pl_stream_t stream) {
  if (!A || !B || !D || M < 1 || N < 1 || K < 1) return PL_ERR_ARG;
  if (M > (1 << 30) || N > (1 << 30) || K > (1 << 30) || ldd < N) return PL_ERR_ARG;
  if (out_path < kOutDirect || out_path > kOutTmaReduce) return PL_ERR_ARG;
  const uint32_t dcode = (mode & PL_DTYPE_MASK) >> 4;
  if (dcode != 1 && dcode != 2) return PL_ERR_DTYPE;
  if (mode & ~PL_DTYPE_MASK) return PL_ERR_ARG;
  if ((lda % 8) || (ldb % 8) || (((uintptr_t)A) & 15) || (((uintptr_t)B) & 15)) return PL_ERR_ALIGN;
  // The TMA paths need 16-byte rows: and N * 4 bytes a multiple of 16 as well,
  // since a store was seen to write the whole 16-byte chunk that holds the
  // last column of a row.
  if (out_path != kOutDirect && ((ldd % 4) || (N % 4) || (((uintptr_t)D) & 15))) return PL_ERR_ALIGN;
  if (lda < (a_mn ? M : K) || ldb < (b_mn ? N : K)) return PL_ERR_ARG;
  pl_status st = check_arch();
  if (st != PL_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  void* scratch = nullptr;
  if ((st = own_workspace(s, loss_ws_bytes(0), &scratch, true)) != PL_OK) return st;
  const DType dt = (DType)dcode;
  GemmParams p{};
  p.err = static_cast<unsigned*>(scratch);
  p.wait_ns = kWaitLimitNs;
  bool ok = a_mn ? make_tmap_2d(&p.maps[0], A, dt, M, K, lda * 2, 64, kBK)
                 : make_tmap_2d(&p.maps[0], A, dt, K, M, lda * 2, kBK, kBM);
  ok = ok && (b_mn ? make_tmap_2d(&p.maps[1], B, dt, N, K, ldb * 2, 64, kBK)
                   : make_tmap_2d(&p.maps[1], B, dt, K, N, ldb * 2, kBK, kBNh));
  if (out_path != kOutDirect) ok = ok && make_tmap_2d(&p.maps[4], D, DType::F32, N, M, ldd * 4, kOutBoxN, kOutBoxM);
  if (!ok) return PL_ERR_CUDA;
  GemmJob& j = p.jobs[0];
  j.a_map = 0; j.b_map = 1; j.a_mn = a_mn ? 1 : 0; j.b_mn = b_mn ? 1 : 0;
  j.M = (int)M; j.N = (int)N; j.K = (int)K; j.n_inner = 0; j.epi = kEpiStore;
  j.out = D; j.out_f32 = 1; j.acc_in = nullptr; j.out_ld = ldd; j.scale = nullptr;
  j.out_path = out_path; j.out_map = 4;
  p.njobs = 1;
  gemm_finalize_jobs(&p);
  return launch_gemm(p, dt, s) == cudaSuccess ? PL_OK : PL_ERR_CUDA;
}

extern "C" pl_status pl_debug_gemm(const void* A, int a_mn, int64_t lda, const void* B, int b_mn,
                                   int64_t ldb, float* D, int64_t M, int64_t N, int64_t K, uint32_t mode,
                                   pl_stream_t stream) {
  return pl_debug_gemm_out(A, a_mn, lda, B, b_mn, ldb, D, N, kOutDirect, M, N, K, mode, stream);
}

// pl_debug_pick_tile: the tile width the GEMM launcher picks for one or two
// problems (M, N, K each) on `pairs` CTA pairs.
extern "C" int pl_debug_pick_tile(int njobs, const int64_t* mnk, int pairs) {
  if (njobs < 1 || njobs > 2 || !mnk || pairs < 1) return -1;
  GemmParams p{};
  p.njobs = njobs;
  for (int i = 0; i < njobs; ++i) {
    if (mnk[3 * i] < 1 || mnk[3 * i + 1] < 1 || mnk[3 * i + 2] < 1) return -1;
    if (mnk[3 * i] > (1 << 30) || mnk[3 * i + 1] > (1 << 30) || mnk[3 * i + 2] > (1 << 30)) return -1;
    p.jobs[i].M = (int)mnk[3 * i];
    p.jobs[i].N = (int)mnk[3 * i + 1];
    p.jobs[i].K = (int)mnk[3 * i + 2];
  }
  return pick_tile_width(p, pairs);
}

// pl_debug_pick_split: the K-split choice for the dX problem (job 0) of a
// two-problem backward launch, and the tile width that goes with it.
extern "C" int pl_debug_pick_split(const int64_t* mnk, int pairs, int* nh_out) {
  if (!mnk || pairs < 1) return -1;
  GemmParams p{};
  p.njobs = 2;
  for (int i = 0; i < 2; ++i) {
    if (mnk[3 * i] < 1 || mnk[3 * i + 1] < 1 || mnk[3 * i + 2] < 1) return -1;
    if (mnk[3 * i] > (1 << 30) || mnk[3 * i + 1] > (1 << 30) || mnk[3 * i + 2] > (1 << 30)) return -1;
    p.jobs[i].M = (int)mnk[3 * i];
    p.jobs[i].N = (int)mnk[3 * i + 1];
    p.jobs[i].K = (int)mnk[3 * i + 2];
  }
  const int split = gemm_choose_k_split(&p, 0, pairs);
  if (nh_out) *nh_out = p.nh;
  return split;
}

extern "C" int pl_debug_set_gemm_tail(int mode) {
  if (mode < 0 || mode > 1) return PL_ERR_ARG;
  debug_knobs().gemm_tail = mode;
  return PL_OK;
}

extern "C" int pl_debug_tail_halves(int tiles, int pairs) { return tail_halves(tiles, pairs); }

extern "C" int pl_debug_set_dw_finish(int mode) {
  if (mode < 0 || mode > 2) return PL_ERR_ARG;
  debug_knobs().dw_finish = mode;
  return PL_OK;
}

extern "C" int pl_debug_set_dw_pair(int mode) {
  if (mode < 0 || mode > 2) return PL_ERR_ARG;
  debug_knobs().dw_pair = mode;
  return PL_OK;
}

extern "C" int pl_debug_set_gemm_merge(int mode) {
  if (mode < 0 || mode > 2) return PL_ERR_ARG;
  debug_knobs().gemm_merge = mode;
  return PL_OK;
}

// pl_debug_queue_tiles: the dynamic tile queue's order for jobs of the given
// tile counts (leading jobs [0, q_f0), then jobs [q_f0, q_w) interleaved with
// job q_w; q_w < 0: job order).  out[q] receives the global tile id of entry q.
extern "C" int pl_debug_queue_tiles(int njobs, const int32_t* tiles, int q_f0, int q_w, int32_t* out) {
  if (njobs < 1 || njobs > kMaxJobs || !tiles || !out) return -1;
  if (q_w >= njobs || (q_w >= 0 && (q_f0 < 0 || q_f0 > q_w))) return -1;
  GemmParams p{};
  p.njobs = njobs;
  int begin = 0;
  for (int i = 0; i < njobs; ++i) {
    if (tiles[i] < 0) return -1;
    p.jobs[i].tile_begin = begin;
    begin += tiles[i];
  }
  p.total_tiles = begin;
  p.q_f0 = q_f0;
  p.q_w = q_w;
  for (int q = 0; q < begin; ++q) out[q] = queue_tile(p, q);
  return 0;
}

extern "C" int pl_debug_set_gemm_split(int mode) {
  if (mode < 0 || mode > 2) return PL_ERR_ARG;
  debug_knobs().gemm_split = mode;
  return PL_OK;
}

// pl_debug_pair_tiles: the GEMM's tile schedule for two jobs (t0 tiles of c0
// k-steps, then t1 tiles of c1 k-steps) over `pairs` CTA pairs.  Writes, for
// every tile, the pair that runs it (out_pair[t0 + t1]) and returns 0, or -1 if
// a tile is given to no pair or to two.
extern "C" int pl_debug_pair_tiles(int t0, int t1, int c0, int c1, int pairs, int32_t* out_pair) {
  if (t0 < 0 || t1 < 0 || pairs < 1 || !out_pair) return -1;
  GemmParams p{};
  p.njobs = 2;
  p.jobs[0].tiles_m = t0; p.jobs[0].tiles_n = 1; p.jobs[0].k_steps = c0; p.jobs[0].tile_begin = 0;
  p.jobs[1].tiles_m = t1; p.jobs[1].tiles_n = 1; p.jobs[1].k_steps = c1; p.jobs[1].tile_begin = t0;
  p.total_tiles = t0 + t1;
  balance_schedule(&p, pairs);
  for (int t = 0; t < t0 + t1; ++t) out_pair[t] = -1;
  for (int q = 0; q < pairs; ++q) {
    for (int i = 0;; ++i) {
      const int t = pair_tile(p, q, pairs, i);
      if (t < 0) break;
      if (t >= t0 + t1 || out_pair[t] != -1) return -1;
      out_pair[t] = q;
    }
  }
  for (int t = 0; t < t0 + t1; ++t)
    if (out_pair[t] < 0) return -1;
  return 0;
}

// ---------------------------------------------------------------- launch bookkeeping
#include <atomic>
#include <vector>

namespace {
std::atomic<int64_t> g_launches{0};
bool g_timing = false;
struct EvPair {
  cudaEvent_t a = nullptr, b = nullptr;
  int kind = 0;
};
std::vector<EvPair> g_pool;
size_t g_used = 0;
}  // namespace

namespace pl {
void launch_begin(int kind, cudaStream_t stream) {
  g_launches.fetch_add(1, std::memory_order_relaxed);
  if (!g_timing) return;
  if (g_used == g_pool.size()) {
    EvPair e;
    if (cudaEventCreate(&e.a) != cudaSuccess || cudaEventCreate(&e.b) != cudaSuccess) return;
    g_pool.push_back(e);
  }
  g_pool[g_used].kind = kind;
  cudaEventRecord(g_pool[g_used].a, stream);
}
void launch_end(int kind, cudaStream_t stream) {
  (void)kind;
  if (!g_timing || g_used >= g_pool.size()) return;
  cudaEventRecord(g_pool[g_used].b, stream);
  ++g_used;
}
}  // namespace pl

namespace pl {
DebugKnobs& debug_knobs() {
  static DebugKnobs k;
  return k;
}
}  // namespace pl

extern "C" int pl_debug_set_loss_path(int path) {
  if (path < 0 || path > 2) return PL_ERR_ARG;
  debug_knobs().loss_path = path;
  return PL_OK;
}

extern "C" void pl_debug_set_wait(unsigned long long wait_ns, unsigned extra_arrivals, unsigned extra_tx) {
  DebugKnobs& k = debug_knobs();
  k.wait_ns = wait_ns ? wait_ns : kWaitLimitNs;
  k.extra_arrivals = extra_arrivals;
  k.extra_tx = extra_tx;
}

extern "C" int pl_debug_set_gemm_tile(int nh) {
  if (nh < 0 || nh > 2) return PL_ERR_ARG;
  debug_knobs().gemm_nh = nh;
  return PL_OK;
}

extern "C" int pl_debug_set_rkl_path(int path) {
  if (path < 0 || path > 2) return PL_ERR_ARG;
  debug_knobs().rkl_path = path;
  return PL_OK;
}

extern "C" int pl_debug_set_rkl_cluster(int cl) {
  if (cl != 0 && cl != 1 && cl != 2 && cl != 4 && cl != 8) return PL_ERR_ARG;
  debug_knobs().rkl_cluster = cl;
  return PL_OK;
}

extern "C" void pl_debug_timing(int enable) { g_timing = enable != 0; }

extern "C" pl_status pl_debug_timing_read(double* ms, int64_t* launches) {
  for (int k = 0; k < 3; ++k) {
    if (ms) ms[k] = 0.0;
    if (launches) launches[k] = 0;
  }
  for (size_t i = 0; i < g_used; ++i) {
    float t = 0.0f;
    if (cudaEventSynchronize(g_pool[i].b) != cudaSuccess) return PL_ERR_CUDA;
    if (cudaEventElapsedTime(&t, g_pool[i].a, g_pool[i].b) != cudaSuccess) return PL_ERR_CUDA;
    const int k = g_pool[i].kind;
    if (k >= 0 && k < 3) {
      if (ms) ms[k] += t;
      if (launches) launches[k] += 1;
    }
  }
  g_used = 0;
  return PL_OK;
}

extern "C" int64_t pl_debug_launch_count(void) { return g_launches.load(); }
