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
  int64_t N = 0, C = 1024, Cbuf = 1, nchunks = 0, ld = 0;
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
  p.off.logits = region(2 * p.Cbuf * p.ld);
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
  int last_blocks = 0;
  for (int64_t c = 0; c < plan.nchunks; ++c) {
    const int64_t r0 = c * plan.C;
    const int64_t rows = (N - r0) < plan.C ? (N - r0) : plan.C;

    // ---- forward GEMM(s): reference then policy logits tiles ----
    GemmParams fp{};
    fp.err = reinterpret_cast<unsigned*>(ws);
    fp.wait_ns = kWaitLimitNs;
    int nj = 0;
    if (has_kl) {
      if (!make_tmap_2d(&fp.maps[0], Xrb + r0 * H * esz, dt, H, rows, H * esz, kBK, kBM) ||
          !make_tmap_2d(&fp.maps[1], Wref, dt, H, V, H * esz, kBK, kBNh))
        return PL_ERR_CUDA;
      GemmJob& j = fp.jobs[nj++];
      j.a_map = 0; j.b_map = 1; j.a_mn = 0; j.b_mn = 0;
      j.M = (int)rows; j.N = (int)V; j.K = (int)H; j.n_inner = 0; j.epi = kEpiLse;
      j.bias = nullptr; j.targets = targets + r0;
      j.part = reinterpret_cast<float2*>(ws + plan.off.part_ref); j.part_ld = plan.nparts;
      j.zt = reinterpret_cast<float*>(ws + plan.off.zt_ref); j.logits = nullptr;
      j.logit_scale = q.inv_temp;
    }
    if (!make_tmap_2d(&fp.maps[2], Xb + r0 * H * esz, dt, H, rows, H * esz, kBK, kBM) ||
        !make_tmap_2d(&fp.maps[3], W, dt, H, V, H * esz, kBK, kBNh))
      return PL_ERR_CUDA;
    {
      GemmJob& j = fp.jobs[nj++];
      j.a_map = 2; j.b_map = 3; j.a_mn = 0; j.b_mn = 0;
      j.M = (int)rows; j.N = (int)V; j.K = (int)H; j.n_inner = 0; j.epi = kEpiLse;
      j.bias = bias; j.targets = targets + r0;
      j.part = reinterpret_cast<float2*>(ws + plan.off.part); j.part_ld = plan.nparts;
      j.zt = reinterpret_cast<float*>(ws + plan.off.zt);
      j.logits = need_bwd ? ws + plan.off.logits : nullptr; j.logits_ld = plan.ld;
      j.logit_scale = q.inv_temp;
      if (j.logits) {
        // the chunk's [rows, V] logits, written by TMA stores from the epilogue
        if (!make_tmap_2d(&fp.maps[4], ws + plan.off.logits, dt, V, rows, plan.ld * esz, kOutBoxN16, kOutBoxM))
          return PL_ERR_CUDA;
        j.out_path = kOutTmaStore; j.out_map = 4;
      }
    }
    fp.njobs = nj;
    gemm_finalize_jobs(&fp);
    if (!ok(launch_gemm(fp, dt, s))) return PL_ERR_CUDA;

    // ---- combine: lse, logp, loss partials, g ----
    CombineArgs ca{};
    ca.ws = ws; ca.off = plan.off; ca.targets = targets; ca.old_lp = old_lp; ca.adv = adv; ca.mask = mask;
    ca.logp_out = logp_out; ca.ref_logp_out = ref_logp_out;
    ca.row0 = r0; ca.rows = rows; ca.bs = bs; ca.T = T; ca.V = V; ca.nparts = plan.nparts;
    ca.chunk = (int)c; ca.part_stride = plan.part_stride;
    ca.lo = 1.0f - eps_lo; ca.hi = 1.0f + eps_hi; ca.beta = beta;
    ca.grpo = (mode & PL_REDUCTION_MASK) == PL_GRPO; ca.adv_lp_dtype = (mode & PL_ADV_LP_DTYPE) != 0;
    ca.bf16 = dt == DType::BF16;
    ca.grad_logp = q.grad_logp;
    ca.g_scale = q.inv_temp;
    if (q.ext_g) {
      if (!ok(launch_combine_ext(ca, s))) return PL_ERR_CUDA;
    } else if (!ok(launch_combine(ca, has_kl, two_sided, s))) {
      return PL_ERR_CUDA;
    }
    last_blocks = (int)((rows + 7) / 8);

    if (!need_bwd) continue;

    // ---- dlogits in place (+ dbias) ----
    DlogitsArgs da{};
    da.ws = ws; da.off = plan.off; da.targets = targets; da.logits = ws + plan.off.logits; da.ld = plan.ld;
    da.row0 = r0; da.rows = rows; da.V = V; da.chunk = (int)c;
    da.dbias_mode = dbias ? acc_mode(c, plan.nchunks) : kAccNone;
    da.dbias_acc = reinterpret_cast<float*>(ws + plan.off.db_acc); da.dbias = dbias;
    da.db_part = reinterpret_cast<float*>(ws + plan.off.db_part);
    da.db_cnt = reinterpret_cast<unsigned*>(ws + plan.off.db_cnt);
    if (!ok(launch_dlogits(da, dt, s))) return PL_ERR_CUDA;

    if (!dX && !dW) continue;

    // ---- backward GEMMs: dX rows of this chunk, dW contribution ----
    GemmParams bp{};
    bp.err = reinterpret_cast<unsigned*>(ws);
    bp.wait_ns = kWaitLimitNs;
    nj = 0;
    const float* inv_scale = reinterpret_cast<const float*>(ws + plan.off.inv_scale) + c;
    if (dX) {
      if (!make_tmap_2d(&bp.maps[0], ws + plan.off.logits, dt, V, rows, plan.ld * esz, kBK, kBM) ||
          !make_tmap_2d(&bp.maps[1], W, dt, H, V, H * esz, 64, kBK))
        return PL_ERR_CUDA;
      GemmJob& j = bp.jobs[nj++];
      j.a_map = 0; j.b_map = 1; j.a_mn = 0; j.b_mn = 1;
      j.M = (int)rows; j.N = (int)H; j.K = (int)V; j.n_inner = 0; j.epi = kEpiStore;
      j.out = static_cast<unsigned char*>(dX) + r0 * H * esz; j.out_f32 = 0; j.acc_in = nullptr;
      j.out_ld = H; j.scale = inv_scale;
      // whole 128-byte lines through the TMA unit when dX is 16-byte aligned
      if (aligned(dX, 16)) {
        if (!make_tmap_2d(&bp.maps[5], j.out, dt, H, rows, H * esz, kOutBoxN16, kOutBoxM)) return PL_ERR_CUDA;
        j.out_path = kOutTmaStore; j.out_map = 5;
      }
    }
    if (dW) {
      if (!make_tmap_2d(&bp.maps[2], ws + plan.off.logits, dt, V, rows, plan.ld * esz, 64, kBK) ||
          !make_tmap_2d(&bp.maps[3], Xb + r0 * H * esz, dt, H, rows, H * esz, 64, kBK))
        return PL_ERR_CUDA;
      GemmJob& j = bp.jobs[nj++];
      j.a_map = 2; j.b_map = 3; j.a_mn = 1; j.b_mn = 1;
      j.M = (int)V; j.N = (int)H; j.K = (int)rows; j.n_inner = 1; j.epi = kEpiStore;
      j.out_ld = H; j.scale = inv_scale;
      // Several chunks: the first stores its fp32 contribution, every later one
      // adds its own through the TMA unit (the memory system does the add, so
      // the epilogue never waits on a load), and the sum is rounded to the
      // model dtype once, after the last chunk.
      float* acc = reinterpret_cast<float*>(ws + plan.off.dw_acc);
      j.acc_in = nullptr;
      if (plan.nchunks == 1) {
        j.out = dW; j.out_f32 = 0; j.out_path = kOutDirect;
        if (aligned(dW, 16)) {
          if (!make_tmap_2d(&bp.maps[4], dW, dt, H, V, H * esz, kOutBoxN16, kOutBoxM)) return PL_ERR_CUDA;
          j.out_path = kOutTmaStore; j.out_map = 4;
        }
      } else {
        if (!make_tmap_2d(&bp.maps[4], acc, DType::F32, H, V, H * 4, kOutBoxN, kOutBoxM)) return PL_ERR_CUDA;
        j.out = acc; j.out_f32 = 1; j.out_map = 4;
        j.out_path = c == 0 ? kOutTmaStore : kOutTmaReduce;
      }
    }
    bp.njobs = nj;
    gemm_finalize_jobs(&bp);
    // dX has K = V: its few long tiles would finish last next to the many short
    // dW tiles.  When the schedule estimate says so, each dX tile is computed as
    // two tiles over the halves of the vocabulary, both adding their fp32 result
    // into a zeroed buffer through the TMA unit (two addends onto zero: the sum
    // does not depend on their order), which one pass then rounds into dX.
    int dx_split = 1;
    float* dx_acc = reinterpret_cast<float*>(ws + plan.off.dx_acc);
    if (dX) {
      DevInfo di;
      if (dev_info(&di) != cudaSuccess) return PL_ERR_CUDA;
      dx_split = gemm_choose_k_split(&bp, 0, di.sm_count / 2);
    }
    if (dx_split == 2) {
      GemmJob& j = bp.jobs[0];
      if (!make_tmap_2d(&bp.maps[5], dx_acc, DType::F32, H, rows, H * 4, kOutBoxN, kOutBoxM)) return PL_ERR_CUDA;
      j.out = dx_acc; j.out_f32 = 1; j.out_path = kOutTmaReduce; j.out_map = 5; j.out_ld = H;
      if (!ok(cudaMemsetAsync(dx_acc, 0, (size_t)rows * H * 4, s))) return PL_ERR_CUDA;
    }
    if (!ok(launch_gemm(bp, dt, s))) return PL_ERR_CUDA;
    if (dx_split == 2 &&
        !ok(launch_convert(dx_acc, static_cast<unsigned char*>(dX) + r0 * H * esz, rows * H, dt, s)))
      return PL_ERR_CUDA;
    if (dW && plan.nchunks > 1 && c + 1 == plan.nchunks &&
        !ok(launch_convert(reinterpret_cast<const float*>(ws + plan.off.dw_acc), dW, V * H, dt, s)))
      return PL_ERR_CUDA;
  }

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
