// Plain CPU oracle for the fused GRPO/BNPO policy loss (TEST INFRASTRUCTURE).
//
// This file is the slow, obviously-correct fp64 statement of what the GPU path
// computes. Only the test-suite, the smoke check and the CPU-baseline leg of the
// benchmark may load it; the product library never links, imports or calls it,
// and it shares no code, header or constant with the CUDA sources.
//
// What it computes, and where each step is defined:
//   * policy_loss   -- the PPO-clipped per-token loss, the k3 KL penalty and the
//                      BNPO / GRPO reductions of the "Geometric-AI Kernels" model
//                      card, sections "BNPO Loss" and "GRPO Loss"; the gradient
//                      with respect to the policy log-probs is the analytic
//                      derivative of that loss (the card's fused forward+backward
//                      returns (loss, grad_logprobs)).
//   * lm_head_logprob -- selective log-probability: z = (X W^T (+ b)) / temperature,
//                      logp = z[target] - logsumexp(z), as used by "Add SM100 CuTe
//                      DSL GRPO fast path" (Liger-Kernel PR #1363), "Summary" and
//                      "Native scope" (temperature 1.0 natively, other temperatures
//                      handled by the page's older path).
//   * lm_head_backward -- the chain rule through log-softmax and the linear layer:
//                      dz = g * (onehot(target) - softmax(z)), dX = dz W,
//                      dW = dz^T X, dbias = sum over rows of dz.
//   * reverse_kl    -- reverse-KL self-distillation of the "Geometric-AI Kernels"
//                      model card, section "Reverse KL": p = softmax(student row),
//                      q = softmax(teacher row), kl_r = sum_v p_v (log p_v - log q_v),
//                      loss = sum_r mask_r kl_r / n_valid, and the gradient with
//                      respect to the student logits
//                      mask_r / n_valid * p_v (log p_v - log q_v - kl_r).
//
// Everything is fp64.  Low-precision inputs (binary16, bfloat16, binary32) are
// decoded exactly by the decoders below, written from the IEEE-754 / bfloat16
// bit-layout definitions.  Contractions are plain sums taken in natural index
// order; the only concession to speed is that 32 rows share one pass over a
// weight row, their 32 sums held in vector registers (each sum is still its own
// accumulator, taken in the same h order).
//
// Readings of points the pages leave open (each also listed in the design notes):
//   * clip bounds mirror fp32 arguments: lo = (double)(1.0f - eps_lo),
//     hi = (double)(1.0f + eps_hi);
//   * default clip form is the literal one, -A * min(r, clip(r, lo, hi)); its
//     gradient is -A*r when r <= hi and 0 otherwise (ties flow);
//   * optional two-sided form -min(A*r, A*clip(r)); gradient -A*r when
//     A*r <= A*clip(r), else 0;
//   * a mask entry counts as valid when it is nonzero;
//   * GRPO divides by bs, counting fully masked rows (which contribute 0).
//   * reverse KL divides by max(n_valid, 1): the card leaves the all-masked
//     batch undefined (inf/NaN); clamping makes it loss 0, gradient 0, and
//     changes nothing when any row is valid.

#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>
#include <algorithm>
#include <sched.h>

namespace {

enum { DT_F64 = 0, DT_F32 = 1, DT_F16 = 2, DT_BF16 = 3 };

// binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits.
double decode_f16(uint16_t b) {
  const int sign = (b >> 15) & 1;
  const int e = (b >> 10) & 0x1f;
  const int f = b & 0x3ff;
  double v;
  if (e == 0) {
    v = std::ldexp((double)f, -24);                 // subnormal: f * 2^-24
  } else if (e == 31) {
    v = f ? NAN : INFINITY;
  } else {
    v = std::ldexp((double)(1024 + f), e - 25);     // (1 + f/1024) * 2^(e-15)
  }
  return sign ? -v : v;
}

// bfloat16 is the upper half of a binary32 word.
double decode_bf16(uint16_t b) {
  uint32_t w = (uint32_t)b << 16;
  float f;
  std::memcpy(&f, &w, 4);
  return (double)f;
}

double load(int dt, const void* p, int64_t i) {
  switch (dt) {
    case DT_F64: return ((const double*)p)[i];
    case DT_F32: return (double)((const float*)p)[i];
    case DT_F16: return decode_f16(((const uint16_t*)p)[i]);
    case DT_BF16: return decode_bf16(((const uint16_t*)p)[i]);
  }
  return NAN;
}

// dst[i] = exact value of element (off + i) for i < n; the dtype switch is
// taken once per row rather than once per element.
void load_row(int dt, const void* p, int64_t off, int64_t n, double* dst) {
  switch (dt) {
    case DT_F64: for (int64_t i = 0; i < n; ++i) dst[i] = ((const double*)p)[off + i]; break;
    case DT_F32: for (int64_t i = 0; i < n; ++i) dst[i] = (double)((const float*)p)[off + i]; break;
    case DT_F16: for (int64_t i = 0; i < n; ++i) dst[i] = decode_f16(((const uint16_t*)p)[off + i]); break;
    case DT_BF16: for (int64_t i = 0; i < n; ++i) dst[i] = decode_bf16(((const uint16_t*)p)[off + i]); break;
    default: for (int64_t i = 0; i < n; ++i) dst[i] = NAN;
  }
}

int worker_count(int requested) {
  if (requested > 0) return requested;
  cpu_set_t set;
  if (sched_getaffinity(0, sizeof(set), &set) == 0) {
    int n = CPU_COUNT(&set);
    if (n > 0) return n;
  }
  unsigned n = std::thread::hardware_concurrency();
  return n ? (int)n : 1;
}

// acc[r] = sum over h (in order h = 0..H-1) of xT[h*32 + r] * w[h], for the 32
// rows of a group: the same per-row sums as 32 separate dot products, written
// with four-wide vector registers so the accumulators stay in registers.
typedef double v4d __attribute__((vector_size(32), aligned(8)));
void dot32(const double* xT, const double* w, int64_t H, double* acc) {
  v4d a0 = {0, 0, 0, 0}, a1 = a0, a2 = a0, a3 = a0, a4 = a0, a5 = a0, a6 = a0, a7 = a0;
  for (int64_t h = 0; h < H; ++h) {
    const v4d wv = {w[h], w[h], w[h], w[h]};
    const v4d* x = reinterpret_cast<const v4d*>(xT + h * 32);
    a0 += x[0] * wv;
    a1 += x[1] * wv;
    a2 += x[2] * wv;
    a3 += x[3] * wv;
    a4 += x[4] * wv;
    a5 += x[5] * wv;
    a6 += x[6] * wv;
    a7 += x[7] * wv;
  }
  const v4d* all[8] = {&a0, &a1, &a2, &a3, &a4, &a5, &a6, &a7};
  for (int q = 0; q < 8; ++q)
    for (int j = 0; j < 4; ++j) acc[4 * q + j] = (*all[q])[j];
}

// The same for a group of at most 4 rows (xT holds 32 slots per h; only the
// first 4 are read), so small groups do not pay for 32.
void dot4(const double* xT, const double* w, int64_t H, double* acc) {
  v4d a0 = {0, 0, 0, 0};
  for (int64_t h = 0; h < H; ++h) {
    const v4d wv = {w[h], w[h], w[h], w[h]};
    a0 += *reinterpret_cast<const v4d*>(xT + h * 32) * wv;
  }
  for (int j = 0; j < 4; ++j) acc[j] = a0[j];
}

// Runs fn(worker, begin, end) over [0, n) split into contiguous ranges.
template <class F>
void parallel_ranges(int64_t n, int workers, F fn) {
  if (n <= 0) return;
  workers = (int)std::min<int64_t>(workers, n);
  if (workers <= 1) { fn(0, (int64_t)0, n); return; }
  std::vector<std::thread> ts;
  for (int w = 0; w < workers; ++w) {
    int64_t b = n * w / workers, e = n * (w + 1) / workers;
    ts.emplace_back([=] { fn(w, b, e); });
  }
  for (auto& t : ts) t.join();
}

}  // namespace

extern "C" {

int orc_threads(int requested) { return worker_count(requested); }

// Exact decode of n elements of dtype dt into fp64.
int orc_decode(int dt, const void* src, int64_t n, double* dst) {
  if (dt < 0 || dt > 3 || (n > 0 && (!src || !dst))) return 1;
  for (int64_t i = 0; i < n; ++i) dst[i] = load(dt, src, i);
  return 0;
}

// Per-token PPO-clipped loss with k3 KL, BNPO or GRPO reduction, and its
// gradient with respect to the policy log-probs.
//   lp, old_lp, ref_lp : [bs*seq] fp64 (ref_lp may be NULL only when beta == 0)
//   adv                : [bs] fp64
//   mask               : [bs*seq] bytes, nonzero = valid
//   reduction          : 0 = BNPO (global token mean), 1 = GRPO (per-sequence
//                        mean, then mean over the bs sequences)
//   two_sided          : 0 = literal -A*min(r, clip(r)), 1 = -min(A*r, A*clip(r))
// Outputs: loss (scalar), grad [bs*seq] or NULL, n_valid, row_valid [bs] or
// NULL, abs_sum = sum of |scaled per-token contributions| (for relative errors).
int orc_policy_loss(const double* lp, const double* old_lp, const double* ref_lp,
                    const double* adv, const uint8_t* mask, int64_t bs, int64_t seq,
                    float eps_lo, float eps_hi, double beta, int reduction, int two_sided,
                    double* loss, double* grad, int64_t* n_valid, int64_t* row_valid,
                    double* abs_sum) {
  if (bs < 0 || seq < 0 || !loss) return 1;
  if (bs * seq > 0 && (!lp || !old_lp || !adv || !mask)) return 1;
  if (beta != 0.0 && bs * seq > 0 && !ref_lp) return 1;
  if (reduction != 0 && reduction != 1) return 1;

  const double lo = (double)(1.0f - eps_lo);
  const double hi = (double)(1.0f + eps_hi);

  // Valid-token counts: per sequence and over the whole batch.
  std::vector<int64_t> rows(bs > 0 ? bs : 1, 0);
  int64_t total = 0;
  for (int64_t b = 0; b < bs; ++b) {
    int64_t c = 0;
    for (int64_t t = 0; t < seq; ++t) c += mask[b * seq + t] != 0 ? 1 : 0;
    rows[b] = c;
    total += c;
  }

  double loss_acc = 0.0, abs_acc = 0.0;
  for (int64_t b = 0; b < bs; ++b) {
    const double A = adv[b];
    double row_sum = 0.0, row_abs = 0.0;
    // Scale applied to a token's contribution by the reduction.
    const double scale = reduction == 0
        ? 1.0 / (double)std::max<int64_t>(total, 1)
        : 1.0 / ((double)bs * (double)std::max<int64_t>(rows[b], 1));
    for (int64_t t = 0; t < seq; ++t) {
      const int64_t i = b * seq + t;
      const double m = mask[i] != 0 ? 1.0 : 0.0;

      // ratio, clipped ratio and the per-token policy term.
      const double ratio = std::exp(lp[i] - old_lp[i]);
      const double clipped = std::min(std::max(ratio, lo), hi);
      double per_token, dper_token;
      if (!two_sided) {
        per_token = -A * std::min(ratio, clipped);
        dper_token = ratio <= hi ? -A * ratio : 0.0;
      } else {
        per_token = -std::min(A * ratio, A * clipped);
        dper_token = (A * ratio <= A * clipped) ? -A * ratio : 0.0;
      }

      // k3 KL estimator, e = ref - lp.
      double kl = 0.0, dkl = 0.0;
      if (beta != 0.0) {
        const double e = ref_lp[i] - lp[i];
        kl = std::exp(e) - e - 1.0;
        dkl = -std::exp(e) + 1.0;             // d kl / d lp
      }

      const double term = (per_token + beta * kl) * m;
      row_sum += term;
      row_abs += std::fabs(term);
      if (grad) grad[i] = m * (dper_token + beta * dkl) * scale;
    }
    if (reduction == 0) {
      loss_acc += row_sum;
      abs_acc += row_abs;
    } else {
      loss_acc += row_sum / (double)std::max<int64_t>(rows[b], 1);
      abs_acc += row_abs / (double)std::max<int64_t>(rows[b], 1);
    }
    if (row_valid) row_valid[b] = rows[b];
  }
  if (reduction == 0) {
    *loss = loss_acc / (double)std::max<int64_t>(total, 1);
    if (abs_sum) *abs_sum = abs_acc / (double)std::max<int64_t>(total, 1);
  } else {
    *loss = bs > 0 ? loss_acc / (double)bs : 0.0;
    if (abs_sum) *abs_sum = bs > 0 ? abs_acc / (double)bs : 0.0;
  }
  if (n_valid) *n_valid = total;
  return 0;
}

// Selective log-probability: for each selected row i,
//   z_v = (sum_h X[i,h] * W[v,h] (+ bias[v])) / temperature,
//   lse = M + log(sum_v exp(z_v - M)),   logp = z[target_i] - lse.
//   X [N,H] (dtype xdt), W [V,H] (wdt), bias [V] (bdt) or NULL, targets [N].
//   rows: indices of the rows to evaluate (NULL = all N rows, in order).
// Writes lse_out[k], logp_out[k] and, if ztgt_out, the target logit, for the
// k-th selected row.  Returns 2 if a selected target lies outside [0, V).
int orc_lm_head_logprob(const void* X, int xdt, const void* W, int wdt,
                        const void* bias, int bdt, const int64_t* targets,
                        const int64_t* rows, int64_t nsel, int64_t N, int64_t H,
                        int64_t V, int nthreads, double temperature, double* lse_out,
                        double* logp_out, double* ztgt_out) {
  if (!(temperature > 0.0)) return 1;
  if (!X || !W || !targets || !lse_out || !logp_out || H <= 0 || V <= 0) return 1;
  if (!rows) nsel = N;
  const int workers = worker_count(nthreads);
  const int R = 32;                                  // rows sharing one pass over W
  std::vector<double> xT((size_t)H * R);
  std::vector<double> z((size_t)R * V);
  for (int64_t g0 = 0; g0 < nsel; g0 += R) {
    const int gr = (int)std::min<int64_t>(R, nsel - g0);
    int64_t idx[32];
    for (int r = 0; r < gr; ++r) {
      idx[r] = rows ? rows[g0 + r] : g0 + r;
      if (idx[r] < 0 || idx[r] >= N) return 1;
      if (targets[idx[r]] < 0 || targets[idx[r]] >= V) return 2;
    }
    std::fill(xT.begin(), xT.end(), 0.0);
    for (int r = 0; r < gr; ++r)
      for (int64_t h = 0; h < H; ++h) xT[(size_t)h * R + r] = load(xdt, X, idx[r] * H + h);

    parallel_ranges(V, workers, [&](int, int64_t vb, int64_t ve) {
      std::vector<double> w(H);
      double acc[32];
      for (int64_t v = vb; v < ve; ++v) {
        load_row(wdt, W, v * H, H, w.data());
        if (gr <= 4) dot4(xT.data(), w.data(), H, acc); else dot32(xT.data(), w.data(), H, acc);
        const double b = bias ? load(bdt, bias, v) : 0.0;
        for (int r = 0; r < gr; ++r) z[(size_t)r * V + v] = (acc[r] + b) / temperature;
      }
    });

    for (int r = 0; r < gr; ++r) {
      const double* zr = &z[(size_t)r * V];
      double M = -INFINITY;
      for (int64_t v = 0; v < V; ++v) M = std::max(M, zr[v]);
      double S = 0.0;
      for (int64_t v = 0; v < V; ++v) S += std::exp(zr[v] - M);
      const double lse = M + std::log(S);
      const double zt = zr[targets[idx[r]]];
      lse_out[g0 + r] = lse;
      logp_out[g0 + r] = zt - lse;
      if (ztgt_out) ztgt_out[g0 + r] = zt;
    }
  }
  return 0;
}

// Backward through log-softmax, the temperature and the linear layer.
//   lse [N], g [N]: per-row logsumexp and dLoss/dlogp for ALL N rows.
//   dz[i,v] = g_i * ([v == target_i] - exp(z_iv - lse_i)) / temperature
//   (the gradient with respect to the raw logit X W^T + b)
//   dX rows : for each index in dx_rows (n_dx of them)  dX[i,:] = sum_v dz[i,v] W[v,:]
//   dW rows : for each vocab index in dw_rows (n_dw)    dW[v,:] = sum_i dz[i,v] X[i,:]
//             and dbias[v] = sum_i dz[i,v]
// Outputs are [n_dx,H], [n_dw,H], [n_dw] fp64 (any may be NULL with count 0).
int orc_lm_head_backward(const void* X, int xdt, const void* W, int wdt,
                         const void* bias, int bdt, const int64_t* targets,
                         const double* lse, const double* g, int64_t N, int64_t H,
                         int64_t V, int nthreads, double temperature, const int64_t* dx_rows,
                         int64_t n_dx, double* dX_out, const int64_t* dw_rows, int64_t n_dw,
                         double* dW_out, double* dbias_out) {
  if (!(temperature > 0.0)) return 1;
  if (!X || !W || !targets || !lse || !g || H <= 0 || V <= 0 || N < 0) return 1;
  const int workers = worker_count(nthreads);

  // ---- dX rows: groups of R rows share one pass over W -------------------
  if (n_dx > 0) {
    if (!dx_rows || !dX_out) return 1;
    const int R = 32;
    std::vector<double> xT((size_t)H * R);
    for (int64_t g0 = 0; g0 < n_dx; g0 += R) {
      const int gr = (int)std::min<int64_t>(R, n_dx - g0);
      int64_t idx[32];
      for (int r = 0; r < gr; ++r) {
        idx[r] = dx_rows[g0 + r];
        if (idx[r] < 0 || idx[r] >= N) return 1;
      }
      std::fill(xT.begin(), xT.end(), 0.0);
      for (int r = 0; r < gr; ++r)
        for (int64_t h = 0; h < H; ++h) xT[(size_t)h * R + r] = load(xdt, X, idx[r] * H + h);
      const int nw = (int)std::min<int64_t>(workers, V);
      std::vector<std::vector<double>> part(nw, std::vector<double>((size_t)gr * H, 0.0));
      parallel_ranges(V, nw, [&](int wk, int64_t vb, int64_t ve) {
        std::vector<double> w(H);
        double acc[32];
        std::vector<double>& dxp = part[wk];
        for (int64_t v = vb; v < ve; ++v) {
          load_row(wdt, W, v * H, H, w.data());
          if (gr <= 4) dot4(xT.data(), w.data(), H, acc); else dot32(xT.data(), w.data(), H, acc);
          const double b = bias ? load(bdt, bias, v) : 0.0;
          for (int r = 0; r < gr; ++r) {
            const int64_t i = idx[r];
            if (g[i] == 0.0) continue;               // dz row is exactly zero
            const double p = std::exp((acc[r] + b) / temperature - lse[i]);
            // dLoss/d(raw logit) = dLoss/dz / temperature, z = raw / temperature
            const double dz = g[i] * ((v == targets[i] ? 1.0 : 0.0) - p) / temperature;
            double* out = &dxp[(size_t)r * H];
            for (int64_t h = 0; h < H; ++h) out[h] += dz * w[h];
          }
        }
      });
      for (int r = 0; r < gr; ++r)
        for (int64_t h = 0; h < H; ++h) {
          double s = 0.0;
          for (int wk = 0; wk < nw; ++wk) s += part[wk][(size_t)r * H + h];
          dX_out[(g0 + r) * H + h] = s;
        }
    }
  }

  // ---- dW / dbias rows: one vocab row at a time, all N rows --------------
  // z[i, v] for all rows i comes from the same 32-row group dot products as the
  // forward (each z still summed over h in order).
  if (n_dw > 0) {
    if (!dw_rows || !dW_out) return 1;
    std::vector<double> Xd((size_t)N * H);
    for (int64_t i = 0; i < N; ++i) load_row(xdt, X, i * H, H, &Xd[(size_t)i * H]);
    const int64_t ng = (N + 31) / 32;
    std::vector<double> XT((size_t)ng * H * 32, 0.0);
    for (int64_t i = 0; i < N; ++i)
      for (int64_t h = 0; h < H; ++h) XT[(size_t)(i / 32) * H * 32 + (size_t)h * 32 + (i % 32)] = Xd[(size_t)i * H + h];
    for (int64_t k = 0; k < n_dw; ++k)
      if (dw_rows[k] < 0 || dw_rows[k] >= V) return 1;
    parallel_ranges(n_dw, workers, [&](int, int64_t kb, int64_t ke) {
      std::vector<double> w(H);
      double acc[32];
      for (int64_t k = kb; k < ke; ++k) {
        const int64_t v = dw_rows[k];
        load_row(wdt, W, v * H, H, w.data());
        const double b = bias ? load(bdt, bias, v) : 0.0;
        double* out = &dW_out[k * H];
        for (int64_t h = 0; h < H; ++h) out[h] = 0.0;
        double db = 0.0;
        for (int64_t gi = 0; gi < ng; ++gi) {
          const int gr = (int)std::min<int64_t>(32, N - gi * 32);
          const double* xg = &XT[(size_t)gi * H * 32];
          if (gr <= 4) dot4(xg, w.data(), H, acc); else dot32(xg, w.data(), H, acc);
          for (int r = 0; r < gr; ++r) {
            const int64_t i = gi * 32 + r;
            if (g[i] == 0.0) continue;               // dz row is exactly zero
            const double zi = (acc[r] + b) / temperature;
            const double dz = g[i] * ((v == targets[i] ? 1.0 : 0.0) - std::exp(zi - lse[i])) / temperature;
            const double* xi = &Xd[(size_t)i * H];
            for (int64_t h = 0; h < H; ++h) out[h] += dz * xi[h];
            db += dz;
          }
        }
        if (dbias_out) dbias_out[k] = db;
      }
    });
  }
  return 0;
}

// Reverse-KL self-distillation over N rows of V logits.
//   student, teacher: [N, V] (dtype dt, decoded exactly); mask [N] (nonzero =
//   valid) or NULL (every row valid).
//   Per row, in fp64 and natural v order:
//     log p_v = s_v - lse(s),  log q_v = t_v - lse(t)
//     (lse(x) = M + log(sum_v exp(x_v - M)), M = max_v x_v),
//     kl_r = sum_v p_v (log p_v - log q_v).
//   loss = sum_r [mask_r != 0] kl_r / max(n_valid, 1).
//   grad (if not NULL) [N, V]: [mask_r != 0] / max(n_valid, 1) * p_v * (log p_v - log q_v - kl_r).
//   kl_rows (if not NULL) [N]: kl_r of every row, masked or not.
int orc_reverse_kl(const void* student, const void* teacher, int dt, const uint8_t* mask,
                   int64_t N, int64_t V, int nthreads, double* loss_out, double* grad,
                   double* kl_rows, int64_t* n_valid_out) {
  if (!student || !teacher || !loss_out || N < 0 || V <= 0) return 1;
  int64_t n = 0;
  for (int64_t r = 0; r < N; ++r) n += (!mask || mask[r] != 0) ? 1 : 0;
  const double inv_n = 1.0 / (double)std::max<int64_t>(n, 1);
  std::vector<double> kl(N > 0 ? N : 1, 0.0);
  parallel_ranges(N, worker_count(nthreads), [&](int, int64_t rb, int64_t re) {
    std::vector<double> ls(V), lq(V);
    for (int64_t r = rb; r < re; ++r) {
      load_row(dt, student, r * V, V, ls.data());
      load_row(dt, teacher, r * V, V, lq.data());
      for (std::vector<double>* x : {&ls, &lq}) {
        double M = -INFINITY;
        for (int64_t v = 0; v < V; ++v) M = std::max(M, (*x)[v]);
        double S = 0.0;
        for (int64_t v = 0; v < V; ++v) S += std::exp((*x)[v] - M);
        const double lse = M + std::log(S);
        for (int64_t v = 0; v < V; ++v) (*x)[v] -= lse;
      }
      double k = 0.0;
      for (int64_t v = 0; v < V; ++v) k += std::exp(ls[v]) * (ls[v] - lq[v]);
      kl[r] = k;
      if (grad) {
        const double scale = (!mask || mask[r] != 0) ? inv_n : 0.0;
        double* gr = grad + r * V;
        for (int64_t v = 0; v < V; ++v) gr[v] = scale * std::exp(ls[v]) * (ls[v] - lq[v] - k);
      }
    }
  });
  double sum = 0.0;
  for (int64_t r = 0; r < N; ++r)
    if (!mask || mask[r] != 0) sum += kl[r];
  *loss_out = sum * inv_n;
  if (kl_rows)
    for (int64_t r = 0; r < N; ++r) kl_rows[r] = kl[r];
  if (n_valid_out) *n_valid_out = n;
  return 0;
}

}  // extern "C"
