// Host driver of the fused linear path (pl_fused_linear_grpo): validation,
// workspace layout, tensor maps and the per-chunk launch sequence
//
//   count  ->  for each chunk of <= C rows:
//                GEMM  [reference logits tile -> (max, sum exp), target logit]   (beta != 0)
//                      [policy logits tile    -> same + logits into the workspace]
//                combine  (lse, logp, ref_logp, loss partials, g)
//                dlogits  (in place, 2^e-scaled, + dbias)                       (if a gradient is wanted)
//                GEMM  [dX rows of the chunk = dz W]  [dW (+)= dz^T X_chunk]     (if dX or dW)
//                (convert: dX from its fp32 buffer, when the GEMM split dX's K in two)
//          -> convert (the fp32 dW accumulator to the model dtype; several chunks only)
//          -> finalize (fixed-order loss sum)
//
// following "Add SM100 CuTe DSL GRPO fast path" (Liger-Kernel PR #1363):
// one large GEMM per group of up to 1024 rows instead of many vocabulary blocks,
// a bounded logits workspace, direct log-prob output, and fp32 accumulation of
// the weight/bias gradient across chunks where the first chunk's result becomes
// the accumulator ("Why it is faster and uses less memory").  All work is
// enqueued on the caller's stream; there is no host synchronisation.
#include <cmath>

#include "fused.h"
#include "gemm.h"

namespace pl {
namespace {

int64_t align_up(int64_t x, int64_t a) { return (x + a - 1) / a * a; }

struct Plan {
  int64_t N = 0, C = 1024, Cbuf = 1, nchunks = 0, ld = 0, logits_bytes = 0;
  int nslots = 1;    // chunk-sized slots of the logits region
  bool pair = false; // bf16, dW wanted, several chunks: chunks 2i and 2i+1 share one dW job
  int ntv = 0, nparts = 0, part_stride = 1;  // 256-column vocabulary tiles; LSE partials per row
  FusedOffsets off{};
};

constexpr uint32_t kFusedModeBits =
    PL_REDUCTION_MASK | PL_DTYPE_MASK | PL_ADV_LP_DTYPE | PL_CLIP_TWO_SIDED | (0xFFu << PL_CHUNK_SHIFT);

Plan make_plan(int64_t bs, int64_t T, int64_t H, int64_t V, uint32_t mode, bool need_dW, bool need_dbias) {
  Plan p;
  p.N = bs * T;
  int64_t c = (int64_t)((mode >> PL_CHUNK_SHIFT) & 0xFF) * 128;
  p.C = c > 0 ? c : 1024;
  p.Cbuf = p.N > 0 ? (p.N < p.C ? p.N : p.C) : 1;
  p.nchunks = p.N > 0 ? (p.N + p.C - 1) / p.C : 0;
  p.ntv = (int)((V + kBN - 1) / kBN);
  p.nparts = p.ntv * kEpiColGroups;
  p.ld = align_up(V > 0 ? V : 1, 64);
  p.part_stride = (int)((p.Cbuf + 7) / 8);
  int64_t cur = (int64_t)kWsHeader;
  auto region = [&](int64_t bytes) {
    cur = align_up(cur, 1024);
    const int64_t at = cur;
    cur += bytes > 0 ? bytes : 0;
    return at;
  };
  const int64_t nch = p.nchunks > 0 ? p.nchunks : 1;
  p.off.row_cnt = region(8 * (bs > 0 ? bs : 1));
  p.off.loss_part = region(8 * nch * p.part_stride);
  p.off.gmax = region(4 * nch);
  p.off.inv_scale = region(4 * nch);
  p.off.lse = region(4 * p.Cbuf);
  p.off.g = region(4 * p.Cbuf);
  p.off.zt = region(4 * p.Cbuf);
  p.off.zt_ref = region(4 * p.Cbuf);
  p.off.part = region(8 * p.Cbuf * (int64_t)p.nparts);
  p.off.part_ref = region(8 * p.Cbuf * (int64_t)p.nparts);
  // Several chunks: chunk c's backward and chunk c+1's forward share a launch, so
  // two chunks' logits are live at once (see run_pipeline); with paired dW jobs
  // (bf16 with a weight gradient) chunk 2i's dlogits also wait for chunk 2i+1's,
  // and from three chunks on a third slot takes chunk 2i+2's forward meanwhile.
  p.pair = need_dW && p.nchunks > 1 && ((mode & PL_DTYPE_MASK) == PL_BF16);
  p.nslots = p.nchunks > 1 ? ((p.pair && p.nchunks > 2) ? 3 : 2) : 1;
  p.logits_bytes = align_up(2 * p.Cbuf * p.ld, 1024);
  p.off.logits = region(p.logits_bytes * p.nslots);
  p.off.dw_acc = region((need_dW && p.nchunks > 1) ? 4 * V * H : 0);
  p.off.dx_acc = region(4 * p.Cbuf * (H > 0 ? H : 0));
  p.off.db_acc = region((need_dbias && p.nchunks > 1) ? 4 * V : 0);
  p.off.db_part = region(need_dbias ? 4 * (int64_t)kDlMaxRowGroups * V : 0);
  p.off.db_cnt = region(need_dbias ? 4 * (int64_t)p.ntv : 0);
  p.off.total = align_up(cur, 1024);
  return p;
}

bool aligned(const void* p, uintptr_t a) { return ((uintptr_t)p & (a - 1)) == 0; }
bool finite_nonneg(float x) { return std::isfinite(x) && x >= 0.0f; }

AccMode acc_mode(int64_t chunk, int64_t nchunks) {
  if (nchunks == 1) return kAccStoreModel;
  if (chunk == 0) return kAccStoreF32;
  if (chunk == nchunks - 1) return kAccAddConvert;
  return kAccAddF32;
}

}  // namespace
}  // namespace pl


namespace pl {
namespace {

// Everything the per-chunk pipeline needs.  `ext_g` selects the selective
// log-prob form: no loss, g_i = grad_logp[i] (external), no counts/finalize.
struct Pipe {
  const void* X; const void* W; const void* bias; const int64_t* targets;
  const void* Xref; const void* Wref; const float* old_lp; const void* adv; const uint8_t* mask;
  int64_t bs, T, H, V;
  float eps_lo, eps_hi, beta;
  uint32_t mode;
  float* loss; void* dX; void* dW; void* dbias; float* logp_out; float* ref_logp_out; int64_t* n_valid_out;
  const float* grad_logp;
  bool ext_g;
  float inv_temp;
  void* workspace;
  pl_stream_t stream;
  DType dt;
  Plan plan;
};

pl_status run_pipeline(const Pipe& q) {
  const void* X = q.X; const void* W = q.W; const void* bias = q.bias; const int64_t* targets = q.targets;
  const void* Xref = q.Xref; const void* Wref = q.Wref; const float* old_lp = q.old_lp; const void* adv = q.adv;
  const uint8_t* mask = q.mask;
  const int64_t bs = q.bs, T = q.T, H = q.H, V = q.V, N = bs * T;
  const float eps_lo = q.eps_lo, eps_hi = q.eps_hi, beta = q.beta;
  const uint32_t mode = q.mode;
  float* loss = q.loss; void* dX = q.dX; void* dW = q.dW; void* dbias = q.dbias;
  float* logp_out = q.logp_out; float* ref_logp_out = q.ref_logp_out; int64_t* n_valid_out = q.n_valid_out;
  pl_stream_t stream = q.stream;
  const DType dt = q.dt;
  const Plan& plan = q.plan;
  const bool has_kl = beta != 0.0f && !q.ext_g;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  unsigned char* ws = static_cast<unsigned char*>(q.workspace);
  const size_t esz = 2;
  const bool two_sided = (mode & PL_CLIP_TWO_SIDED) != 0;
  const bool need_bwd = (dX || dW || dbias) && (!q.ext_g || q.grad_logp);
  auto ok = [](cudaError_t e) { return e == cudaSuccess; };

  if (N == 0) {
    if (dW && V > 0 && H > 0 && !ok(cudaMemsetAsync(dW, 0, (size_t)V * H * esz, s))) return PL_ERR_CUDA;
    if (dbias && V > 0 && !ok(cudaMemsetAsync(dbias, 0, (size_t)V * esz, s))) return PL_ERR_CUDA;
    if (q.ext_g) return PL_OK;
    if (!ok(cudaMemsetAsync(ws + 16, 0, 8, s))) return PL_ERR_CUDA;
    if (!ok(launch_finalize(ws, plan.off, 0, plan.part_stride, 0, loss, n_valid_out, s))) return PL_ERR_CUDA;
    return PL_OK;
  }

  if (q.ext_g) {
    if (!ok(launch_clear_gmax(ws, (int)plan.nchunks, plan.off, s))) return PL_ERR_CUDA;
  } else if (!ok(launch_count(mask, bs, T, ws, (int)plan.nchunks, plan.off, s))) {
    return PL_ERR_CUDA;
  }

  const unsigned char* Xb = static_cast<const unsigned char*>(X);
  const unsigned char* Xrb = static_cast<const unsigned char*>(Xref);
  const bool has_gemm_bwd = need_bwd && (dX || dW);
  // Several chunks with a backward GEMM: chunk c's backward and chunk c+1's
  // forward share one launch (their tiles do not depend on each other), so the
  // memory-heavy dW tiles with their fp32 accumulator adds run beside the
  // compute-heavy forward tiles, and each launch's tail is paid once.  The chunks'
  // logits take turns in the logits region's slots (chunk c in slot c mod slots).
  const bool merge = has_gemm_bwd && plan.nchunks > 1 && debug_knobs().gemm_merge != 1;
  // bf16 chunks 2i and 2i+1 contribute to dW through one job whose K runs over both
  // chunks' rows (half the fp32 accumulator traffic and twice the k-steps per dW
  // tile); their dlogits then share the scale 2^0
  const bool pair = merge && dW && plan.pair && debug_knobs().dw_pair != 1;
  const int nslots = merge ? (pair ? plan.nslots : 2) : 1;
  auto logits_of = [&](int64_t c) -> unsigned char* {
    return ws + plan.off.logits + (c % nslots) * plan.logits_bytes;
  };
  // dW contributions: one per chunk, or one per pair of chunks (the last chunk of
  // an odd count alone)
  const int64_t ncontrib = pair ? (plan.nchunks + 1) / 2 : plan.nchunks;
  auto rows_of = [&](int64_t c) -> int64_t { return (N - c * plan.C) < plan.C ? (N - c * plan.C) : plan.C; };
  // Several chunks: the last chunk adds into the fp32 accumulator like the others
  // and a streaming kernel rounds it (at the copy bandwidth).  On request, the
  // last chunk's dW epilogue instead adds the accumulator and stores the model
  // dtype in one pass: measured, its per-thread accumulator loads slowed that
  // launch by about what the rounding kernel costs, or more.
  const bool fuse_finish = debug_knobs().dw_finish == 2;

  // Chunk c's forward jobs (reference, then policy) appended to g; maps from *nm.
  auto add_fwd = [&](GemmParams& g, int64_t c, int& nm) -> bool {
    const int64_t r0 = c * plan.C, rows = rows_of(c);
    if (has_kl) {
      const int ma = nm++, mb = nm++;
      if (!make_tmap_2d(&g.maps[ma], Xrb + r0 * H * esz, dt, H, rows, H * esz, kBK, kBM) ||
          !make_tmap_2d(&g.maps[mb], Wref, dt, H, V, H * esz, kBK, kBNh))
        return false;
      GemmJob& j = g.jobs[g.njobs++];
      j.a_map = ma; j.b_map = mb; j.a_mn = 0; j.b_mn = 0;
      j.M = (int)rows; j.N = (int)V; j.K = (int)H; j.n_inner = 0; j.epi = kEpiLse;
      j.bias = nullptr; j.targets = targets + r0;
      j.part = reinterpret_cast<float2*>(ws + plan.off.part_ref); j.part_ld = plan.nparts;
      j.zt = reinterpret_cast<float*>(ws + plan.off.zt_ref); j.logits = nullptr;
      j.logit_scale = q.inv_temp;
    }
    const int ma = nm++, mb = nm++;
    if (!make_tmap_2d(&g.maps[ma], Xb + r0 * H * esz, dt, H, rows, H * esz, kBK, kBM) ||
        !make_tmap_2d(&g.maps[mb], W, dt, H, V, H * esz, kBK, kBNh))
      return false;
    GemmJob& j = g.jobs[g.njobs++];
    j.a_map = ma; j.b_map = mb; j.a_mn = 0; j.b_mn = 0;
    j.M = (int)rows; j.N = (int)V; j.K = (int)H; j.n_inner = 0; j.epi = kEpiLse;
    j.bias = bias; j.targets = targets + r0;
    j.part = reinterpret_cast<float2*>(ws + plan.off.part); j.part_ld = plan.nparts;
    j.zt = reinterpret_cast<float*>(ws + plan.off.zt);
    j.logits = need_bwd ? logits_of(c) : nullptr; j.logits_ld = plan.ld;
    j.logit_scale = q.inv_temp;
    if (j.logits) {
      // the chunk's [rows, V] logits, written by TMA stores from the epilogue
      const int mo = nm++;
      if (!make_tmap_2d(&g.maps[mo], j.logits, dt, V, rows, plan.ld * esz, kOutBoxN16, kOutBoxM)) return false;
      j.out_path = kOutTmaStore; j.out_map = mo;
    }
    return true;
  };

  // Chunk c's dX job (rows of this chunk = dz W), appended to g.
  auto add_dx = [&](GemmParams& g, int64_t c, int& nm) -> bool {
    const int64_t r0 = c * plan.C, rows = rows_of(c);
    const int ma = nm++, mb = nm++;
    if (!make_tmap_2d(&g.maps[ma], logits_of(c), dt, V, rows, plan.ld * esz, kBK, kBM) ||
        !make_tmap_2d(&g.maps[mb], W, dt, H, V, H * esz, 64, kBK))
      return false;
    GemmJob& j = g.jobs[g.njobs++];
    j.a_map = ma; j.b_map = mb; j.a_mn = 0; j.b_mn = 1;
    j.M = (int)rows; j.N = (int)H; j.K = (int)V; j.n_inner = 0; j.epi = kEpiStore;
    j.out = static_cast<unsigned char*>(dX) + r0 * H * esz; j.out_f32 = 0; j.acc_in = nullptr;
    j.out_ld = H; j.scale = reinterpret_cast<const float*>(ws + plan.off.inv_scale) + c;
    // whole 128-byte lines through the TMA unit when dX is 16-byte aligned
    if (aligned(dX, 16)) {
      const int mo = nm++;
      if (!make_tmap_2d(&g.maps[mo], j.out, dt, H, rows, H * esz, kOutBoxN16, kOutBoxM)) return false;
      j.out_path = kOutTmaStore; j.out_map = mo;
    }
    return true;
  };

  // The dW contribution of chunks c0..c1 (c1 = c0, or c0 + 1 for a pair: K runs over
  // both chunks' rows, in two segments), appended to g.  Several contributions:
  // the first stores its fp32 result, every later one adds its own through the TMA
  // unit (the memory system does the add, so the epilogue never waits on a load),
  // and the sum is rounded to the model dtype once, after the last.
  auto add_dw = [&](GemmParams& g, int64_t c0, int64_t c1, int& nm) -> bool {
    const int64_t r0 = c0 * plan.C, rows0 = rows_of(c0);
    const int64_t rows = rows0 + (c1 > c0 ? rows_of(c1) : 0);
    const int64_t ci = pair ? c0 / 2 : c0;  // index of this contribution
    const int ma = nm++, mb = nm++, mo = nm++;
    if (!make_tmap_2d(&g.maps[ma], logits_of(c0), dt, V, rows0, plan.ld * esz, 64, kBK) ||
        !make_tmap_2d(&g.maps[mb], Xb + r0 * H * esz, dt, H, rows0, H * esz, 64, kBK))
      return false;
    GemmJob& j = g.jobs[g.njobs++];
    j.a_map = ma; j.b_map = mb; j.a_mn = 1; j.b_mn = 1;
    if (c1 > c0) {
      // chunk c1's rows as the second K segment (chunk c0 is a full chunk: C rows, a whole
      // number of k-steps)
      const int ma2 = nm++, mb2 = nm++;
      const int64_t r1 = c1 * plan.C;
      if (!make_tmap_2d(&g.maps[ma2], logits_of(c1), dt, V, rows_of(c1), plan.ld * esz, 64, kBK) ||
          !make_tmap_2d(&g.maps[mb2], Xb + r1 * H * esz, dt, H, rows_of(c1), H * esz, 64, kBK))
        return false;
      j.k_seg = (int)(rows0 / kBK); j.a_map2 = ma2; j.b_map2 = mb2;
    }
    j.M = (int)V; j.N = (int)H; j.K = (int)rows; j.n_inner = 1; j.epi = kEpiStore;
    // a pair's dlogits share the scale 2^0 (unit_scale), so chunk c0's factor serves both
    j.out_ld = H; j.scale = reinterpret_cast<const float*>(ws + plan.off.inv_scale) + c0;
    float* acc = reinterpret_cast<float*>(ws + plan.off.dw_acc);
    j.acc_in = nullptr;
    if (ncontrib == 1) {
      j.out = dW; j.out_f32 = 0; j.out_path = kOutDirect;
      if (aligned(dW, 16)) {
        if (!make_tmap_2d(&g.maps[mo], dW, dt, H, V, H * esz, kOutBoxN16, kOutBoxM)) return false;
        j.out_path = kOutTmaStore; j.out_map = mo;
      }
    } else if (ci + 1 == ncontrib && fuse_finish) {
      // the last contribution: its epilogue adds the accumulator of the earlier ones and
      // rounds the sum to the model dtype in one pass (no separate rounding kernel)
      j.out = dW; j.out_f32 = 0; j.acc_in = acc; j.out_path = kOutDirect;
      if (aligned(dW, 16)) {
        if (!make_tmap_2d(&g.maps[mo], dW, dt, H, V, H * esz, kOutBoxN16, kOutBoxM)) return false;
        j.out_path = kOutTmaStore; j.out_map = mo;
      }
    } else {
      if (!make_tmap_2d(&g.maps[mo], acc, DType::F32, H, V, H * 4, kOutBoxN, kOutBoxM)) return false;
      j.out = acc; j.out_f32 = 1; j.out_map = mo;
      j.out_path = ci == 0 ? kOutTmaStore : kOutTmaReduce;
    }
    return true;
  };

  int last_blocks = 0;
  auto combine = [&](int64_t c) -> bool {
    const int64_t rows = rows_of(c);
    CombineArgs ca{};
    ca.ws = ws; ca.off = plan.off; ca.targets = targets; ca.old_lp = old_lp; ca.adv = adv; ca.mask = mask;
    ca.logp_out = logp_out; ca.ref_logp_out = ref_logp_out;
    ca.row0 = c * plan.C; ca.rows = rows; ca.bs = bs; ca.T = T; ca.V = V; ca.nparts = plan.nparts;
    ca.chunk = (int)c; ca.part_stride = plan.part_stride;
    ca.lo = 1.0f - eps_lo; ca.hi = 1.0f + eps_hi; ca.beta = beta;
    ca.grpo = (mode & PL_REDUCTION_MASK) == PL_GRPO; ca.adv_lp_dtype = (mode & PL_ADV_LP_DTYPE) != 0;
    ca.bf16 = dt == DType::BF16;
    ca.grad_logp = q.grad_logp;
    ca.g_scale = q.inv_temp;
    last_blocks = (int)((rows + 7) / 8);
    return ok(q.ext_g ? launch_combine_ext(ca, s) : launch_combine(ca, has_kl, two_sided, s));
  };
  auto dlogits = [&](int64_t c) -> bool {
    DlogitsArgs da{};
    da.ws = ws; da.off = plan.off; da.targets = targets; da.logits = logits_of(c); da.ld = plan.ld;
    da.row0 = c * plan.C; da.rows = rows_of(c); da.V = V; da.chunk = (int)c;
    da.unit_scale = pair ? 1 : 0;
    da.dbias_mode = dbias ? acc_mode(c, plan.nchunks) : kAccNone;
    da.dbias_acc = reinterpret_cast<float*>(ws + plan.off.db_acc); da.dbias = dbias;
    da.db_part = reinterpret_cast<float*>(ws + plan.off.db_part);
    da.db_cnt = reinterpret_cast<unsigned*>(ws + plan.off.db_cnt);
    return ok(launch_dlogits(da, dt, s));
  };
  auto fresh = [&]() {
    GemmParams g{};
    g.err = reinterpret_cast<unsigned*>(ws);
    g.wait_ns = kWaitLimitNs;
    g.q_w = -1;
    return g;
  };
  // dX has K = V: a test or measurement may ask for each dX tile to be computed
  // as two tiles over the halves of the vocabulary, both adding their fp32
  // result into a zeroed buffer through the TMA unit (two addends onto zero: the
  // sum does not depend on their order), which one pass then rounds into dX.
  float* dx_acc = reinterpret_cast<float*>(ws + plan.off.dx_acc);
  auto launch_backward_alone = [&](GemmParams& bp, int64_t c) -> bool {
    const int64_t r0 = c * plan.C, rows = rows_of(c);
    gemm_finalize_jobs(&bp);
    int dx_split = 1;
    if (dX) {
      DevInfo di;
      if (dev_info(&di) != cudaSuccess) return false;
      dx_split = gemm_choose_k_split(&bp, 0, di.sm_count / 2);
    }
    if (dx_split == 2) {
      GemmJob& j = bp.jobs[0];
      const int mo = kMaxMaps - 1;
      if (!make_tmap_2d(&bp.maps[mo], dx_acc, DType::F32, H, rows, H * 4, kOutBoxN, kOutBoxM)) return false;
      j.out = dx_acc; j.out_f32 = 1; j.out_path = kOutTmaReduce; j.out_map = mo; j.out_ld = H;
      if (!ok(cudaMemsetAsync(dx_acc, 0, (size_t)rows * H * 4, s))) return false;
    }
    if (!ok(launch_gemm(bp, dt, s))) return false;
    if (dx_split == 2 &&
        !ok(launch_convert(dx_acc, static_cast<unsigned char*>(dX) + r0 * H * esz, rows * H, dt, s)))
      return false;
    return true;
  };

  if (!merge) {
    for (int64_t c = 0; c < plan.nchunks; ++c) {
      // ---- forward GEMM(s): reference then policy logits tiles ----
      GemmParams fp = fresh();
      int nm = 0;
      if (!add_fwd(fp, c, nm)) return PL_ERR_CUDA;
      gemm_finalize_jobs(&fp);
      if (!ok(launch_gemm(fp, dt, s))) return PL_ERR_CUDA;
      // ---- combine: lse, logp, loss partials, g ----
      if (!combine(c)) return PL_ERR_CUDA;
      if (!need_bwd) continue;
      // ---- dlogits in place (+ dbias) ----
      if (!dlogits(c)) return PL_ERR_CUDA;
      if (!dX && !dW) continue;
      // ---- backward GEMMs: dX rows of this chunk, dW contribution ----
      GemmParams bp = fresh();
      nm = 0;
      if ((dX && !add_dx(bp, c, nm)) || (dW && !add_dw(bp, c, c, nm))) return PL_ERR_CUDA;
      if (!launch_backward_alone(bp, c)) return PL_ERR_CUDA;
    }
  } else {
    // chunk 0's forward alone, then [backward c + forward c+1] launches
    {
      GemmParams fp = fresh();
      int nm = 0;
      if (!add_fwd(fp, 0, nm)) return PL_ERR_CUDA;
      gemm_finalize_jobs(&fp);
      if (!ok(launch_gemm(fp, dt, s))) return PL_ERR_CUDA;
      if (!combine(0) || !dlogits(0)) return PL_ERR_CUDA;
    }
    for (int64_t c = 0; c < plan.nchunks; ++c) {
      GemmParams g = fresh();
      int nm = 0;
      // the dW contribution this launch carries: chunk c's own, or with pairs that of
      // chunks c-1 and c (c odd), or chunk c's alone (the last of an odd count)
      int64_t w0 = -1, w1 = -1;
      if (dW) {
        if (!pair) w0 = w1 = c;
        else if (c & 1) { w0 = c - 1; w1 = c; }
        else if (c + 1 == plan.nchunks) w0 = w1 = c;
      }
      if (c + 1 < plan.nchunks) {
        // queue order: dX tiles (long, K = V) first, then the next chunk's
        // forward tiles interleaved evenly with the dW tiles
        if (dX && !add_dx(g, c, nm)) return PL_ERR_CUDA;
        g.q_f0 = g.njobs;
        if (!add_fwd(g, c + 1, nm)) return PL_ERR_CUDA;
        if (w0 >= 0) {
          g.q_w = g.njobs;
          if (!add_dw(g, w0, w1, nm)) return PL_ERR_CUDA;
        }
        g.dyn = 1;
        g.ctr = reinterpret_cast<unsigned*>(ws + kWsGemmQueue);
        g.ctr_done = g.ctr + 1;
        bool wide = true;
        for (int i = 0; i < g.njobs; ++i) wide = wide && g.jobs[i].N >= 2 * kBN;
        g.nh = wide ? 2 : 1;
        gemm_finalize_jobs(&g);
        if (!ok(launch_gemm(g, dt, s))) return PL_ERR_CUDA;
        if (!combine(c + 1) || !dlogits(c + 1)) return PL_ERR_CUDA;
      } else {
        if ((dX && !add_dx(g, c, nm)) || (w0 >= 0 && !add_dw(g, w0, w1, nm))) return PL_ERR_CUDA;
        if (!launch_backward_alone(g, c)) return PL_ERR_CUDA;
      }
    }
  }
  if (dW && ncontrib > 1 && !fuse_finish &&
      !ok(launch_convert(reinterpret_cast<const float*>(ws + plan.off.dw_acc), dW, V * H, dt, s)))
    return PL_ERR_CUDA;

  if (q.ext_g) return PL_OK;
  if (!ok(launch_finalize(ws, plan.off, (int)plan.nchunks, plan.part_stride, last_blocks, loss, n_valid_out, s)))
    return PL_ERR_CUDA;
  return PL_OK;
}

}  // namespace
}  // namespace pl

using namespace pl;

extern "C" {

size_t pl_fused_linear_grpo_workspace_bytes(int64_t bs, int64_t T, int64_t H, int64_t V, uint32_t mode,
                                            int need_dW, int need_dbias) {
  if (bs < 0 || T < 0 || H < 0 || V < 0) return 0;
  return (size_t)make_plan(bs, T, H, V, mode, need_dW != 0, need_dbias != 0).off.total;
}

pl_status pl_fused_linear_grpo_temp(const void* X, const void* W, const void* bias, const int64_t* targets,
                                    const void* Xref, const void* Wref, const float* old_lp, const void* adv,
                                    const uint8_t* mask, int64_t bs, int64_t T, int64_t H, int64_t V,
                                    float eps_lo, float eps_hi, float beta, float temperature, uint32_t mode,
                                    float* loss, void* dX, void* dW, void* dbias, float* logp_out,
                                    float* ref_logp_out, int64_t* n_valid_out, void* workspace,
                                    size_t ws_bytes, pl_stream_t stream) {
  if (!std::isfinite(temperature) || !(temperature > 0.0f)) return PL_ERR_ARG;
  // ---------------- host-side validation (no device call) ----------------
  if (bs < 0 || T < 0 || H < 0 || V < 0 || !loss) return PL_ERR_ARG;
  if (T > 0 && bs > INT64_MAX / T) return PL_ERR_ARG;
  if (mode & ~kFusedModeBits) return PL_ERR_ARG;
  if ((mode & PL_REDUCTION_MASK) > PL_GRPO) return PL_ERR_ARG;
  const uint32_t dcode = (mode & PL_DTYPE_MASK) >> 4;
  if (dcode != 1 && dcode != 2) return PL_ERR_DTYPE;
  const DType dt = (DType)dcode;
  if (!finite_nonneg(eps_lo) || !finite_nonneg(eps_hi) || !finite_nonneg(beta) || eps_lo > 1.0f)
    return PL_ERR_ARG;
  const int64_t N = bs * T;
  const bool has_kl = beta != 0.0f;
  if (N > 0) {
    if (!X || !W || !targets || !old_lp || !adv || !mask) return PL_ERR_ARG;
    if (H < 1 || V < 1) return PL_ERR_ARG;
    if (has_kl && (!Xref || !Wref)) return PL_ERR_ARG;
    if (H % 8) return PL_ERR_ALIGN;
    if (H > (1 << 24) || V > (1ll << 31) - 1) return PL_ERR_ARG;
    if (!aligned(X, 16) || !aligned(W, 16) || (has_kl && (!aligned(Xref, 16) || !aligned(Wref, 16))))
      return PL_ERR_ALIGN;
    if (bias && !aligned(bias, 2)) return PL_ERR_ALIGN;
  }
  const Plan plan = make_plan(bs, T, H, V, mode, dW != nullptr, dbias != nullptr);
  if (!workspace || ws_bytes < (size_t)plan.off.total || !aligned(workspace, 256)) return PL_ERR_WORKSPACE;
  pl_status st = check_arch();
  if (st != PL_OK) return st;
  Pipe q{X, W, bias, targets, Xref, Wref, old_lp, adv, mask, bs, T, H, V, eps_lo, eps_hi, beta, mode,
         loss, dX, dW, dbias, logp_out, ref_logp_out, n_valid_out, nullptr, false, 1.0f / temperature,
         workspace, stream, dt, plan};
  return run_pipeline(q);
}

pl_status pl_fused_linear_grpo(const void* X, const void* W, const void* bias, const int64_t* targets,
                               const void* Xref, const void* Wref, const float* old_lp, const void* adv,
                               const uint8_t* mask, int64_t bs, int64_t T, int64_t H, int64_t V,
                               float eps_lo, float eps_hi, float beta, uint32_t mode, float* loss,
                               void* dX, void* dW, void* dbias, float* logp_out, float* ref_logp_out,
                               int64_t* n_valid_out, void* workspace, size_t ws_bytes,
                               pl_stream_t stream) {
  return pl_fused_linear_grpo_temp(X, W, bias, targets, Xref, Wref, old_lp, adv, mask, bs, T, H, V, eps_lo,
                                   eps_hi, beta, 1.0f, mode, loss, dX, dW, dbias, logp_out, ref_logp_out,
                                   n_valid_out, workspace, ws_bytes, stream);
}


pl_status pl_fused_selective_logprob(const void* X, const void* W, const void* bias, const int64_t* targets,
                                     int64_t N, int64_t H, int64_t V, uint32_t mode, const float* grad_logp,
                                     float* logp_out, void* dX, void* dW, void* dbias, void* workspace,
                                     size_t ws_bytes, pl_stream_t stream) {
  if (N < 0 || H < 0 || V < 0) return PL_ERR_ARG;
  if (mode & ~(PL_DTYPE_MASK | (0xFFu << PL_CHUNK_SHIFT))) return PL_ERR_ARG;
  const uint32_t dcode = (mode & PL_DTYPE_MASK) >> 4;
  if (dcode != 1 && dcode != 2) return PL_ERR_DTYPE;
  const DType dt = (DType)dcode;
  if ((dX || dW || dbias) && !grad_logp) return PL_ERR_ARG;
  if (!logp_out && !dX && !dW && !dbias) return PL_ERR_ARG;
  if (N > 0) {
    if (!X || !W || !targets || H < 1 || V < 1) return PL_ERR_ARG;
    if (H % 8) return PL_ERR_ALIGN;
    if (H > (1 << 24) || V > (1ll << 31) - 1) return PL_ERR_ARG;
    if (!aligned(X, 16) || !aligned(W, 16)) return PL_ERR_ALIGN;
    if (bias && !aligned(bias, 2)) return PL_ERR_ALIGN;
  }
  const Plan plan = make_plan(1, N, H, V, mode, dW != nullptr, dbias != nullptr);
  if (!workspace || ws_bytes < (size_t)plan.off.total || !aligned(workspace, 256)) return PL_ERR_WORKSPACE;
  pl_status st = check_arch();
  if (st != PL_OK) return st;
  Pipe q{X, W, bias, targets, nullptr, nullptr, nullptr, nullptr, nullptr, 1, N, H, V, 0.0f, 0.0f, 0.0f,
         mode, nullptr, dX, dW, dbias, logp_out, nullptr, nullptr, grad_logp, true, 1.0f, workspace, stream,
         dt, plan};
  return run_pipeline(q);
}

size_t pl_fused_selective_logprob_workspace_bytes(int64_t N, int64_t H, int64_t V, uint32_t mode, int need_dW,
                                                  int need_dbias) {
  if (N < 0 || H < 0 || V < 0) return 0;
  return (size_t)make_plan(1, N, H, V, mode, need_dW != 0, need_dbias != 0).off.total;
}

}  // extern "C"
