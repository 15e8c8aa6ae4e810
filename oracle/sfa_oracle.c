/*
 * sfa_oracle.c — plain fp64 CPU oracle of the Signal Field Attention operator.
 *
 * TEST INFRASTRUCTURE ONLY: tests/, __graft_entry__.smoke() and bench.py's
 * CPU-baseline leg are its only users.  It shares no code, header, table or
 * helper with the CUDA library.
 *
 * It is the operator's definition, one token at a time, in double precision:
 * no blocking, no running sums, no reordering.  Each step names the passage it
 * follows.  Sources (web pages):
 *   [P1] "Signal Field Attention (SFA)：8KB代码实现4.16倍推理加速与248倍内存压缩"
 *   [P2] "Signal Field Attention (SFA)" (project README page)
 *   [P3] "Dalin Soma SFA基于信号场注意力机制的神经网络推理加速框架"
 *
 * Readings taken where the pages are silent or garbled (each also recorded
 * with the design notes):
 *   - score scale is 1/sqrt(head_dim) (the extracted [P1 §2.1] formula lost
 *     the square root);
 *   - the near window of token t is positions max(0, t-k+1) .. t inclusive;
 *   - "mean(K_hist)" of [P1 §2.1 eq. S_t] is the one key that leaves the
 *     window at this step, K_{t-k}; no key leaves while t < k;
 *   - every state is updated with token t before it is read for token t;
 *   - S is kept per KV head and added, unchanged, to every query head of that
 *     KV head's group (GQA: head h uses KV head h / (n_q/n_kv));
 *   - the ring mean always divides by ring_size over zero-initialised slots,
 *     as the [P3 §2.4] Metal kernel does;
 *   - the vector fed to ring, field and pool is x = O_near + alpha_far * S;
 *   - each cosine norm is clamped below at 1e-12;
 *   - slots are fixed inputs and the pool mixes the raw slots.
 *
 * Pins (tests/test_oracle_pins.py; tests/test_oracle_mutations.py plants
 * mistakes in copies of this file and checks that a pin catches each):
 *   - near field: library softmax attention (full causal while n <= k, and
 *     sliding-window), with GQA;
 *   - far field: the evicted key when gamma_far = 0, and c(1 - gamma^m) for a
 *     constant key stream;
 *   - ring mean, field and fusion: closed forms on a constant value stream;
 *   - pool: basis-vector slots (closed-form softmax), equal slots, zero x, and
 *     generic inputs against library attention with normalised query and keys;
 *   - the whole path against an unrolled formulation (sums over the history
 *     in place of every recurrence) on generic inputs;
 *   - alpha_layer: hand-worked values and both endpoints;
 *   - the printed constants and the calibration table (tests/golden/).
 * No function here is left "parity unpinned".
 */
#include "sfa_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define SFA_ORACLE_NORM_FLOOR 1e-12

double sfa_oracle_alpha_layer(double alpha_base, double cross_decay, int layer, int n_layers) {
  /* [P3 §2.2] alpha_layer = alpha_base * (0.3 + 0.7 * layer_ratio) * decay^layer,
   * with layer_ratio = layer / (n_layers - 1) from [P2 cross-layer decay formula]. */
  double layer_ratio = (n_layers > 1) ? (double)layer / (double)(n_layers - 1) : 0.0;
  return alpha_base * (0.3 + 0.7 * layer_ratio) * pow(cross_decay, (double)layer);
}

static int params_ok(const sfa_oracle_params* p) {
  if (!p) return 0;
  if (p->n_q_heads <= 0 || p->n_kv_heads <= 0 || p->head_dim <= 0) return 0;
  if (p->n_q_heads % p->n_kv_heads != 0) return 0;
  if (p->window_k <= 0 || p->ring_size <= 0 || p->n_slots <= 0) return 0;
  if (!(p->temperature > 0.0)) return 0;
  return 1;
}

/* One token of one stream.  scratch: window_k + 2*n_slots + hidden doubles. */
static void oracle_token(const sfa_oracle_params* p, double alpha_layer,
                         const float* slots, const double* slot_norm,
                         const float* q, const float* k, const float* v,
                         sfa_oracle_stream* st, double* out, double* scratch) {
  const int nq = p->n_q_heads, nkv = p->n_kv_heads, d = p->head_dim;
  const int K = p->window_k, R = p->ring_size, P = p->n_slots;
  const int H = nq * d;
  const int group = nq / nkv;
  const long long t = st->pos;
  const int wslot = (int)(t % K);

  double* s = scratch;              /* [K] near-field scores        */
  double* x = scratch + K;          /* [H] dual-channel output x_t  */
  double* c = x + H;                /* [P] pool logits              */
  double* w = c + P;                /* [P] pool weights             */

  /* (1) Far field [P1 §2.1 eq. S_t]: the key leaving the window this step is
   * the one stored in slot t mod k, i.e. K_{t-k}; fold it into the EWMA. */
  if (t >= K) {
    for (int g = 0; g < nkv; ++g)
      for (int i = 0; i < d; ++i) {
        const double evicted = st->win_k[((size_t)wslot * nkv + g) * d + i];
        double* Sg = &st->S[(size_t)g * d + i];
        *Sg = p->gamma_far * (*Sg) + (1.0 - p->gamma_far) * evicted;
      }
  }

  /* (2) Window append [P1 §2.2, O(k·d) KV]: K_t, V_t go to slot t mod k. */
  for (int g = 0; g < nkv; ++g)
    for (int i = 0; i < d; ++i) {
      st->win_k[((size_t)wslot * nkv + g) * d + i] = (double)k[(size_t)g * d + i];
      st->win_v[((size_t)wslot * nkv + g) * d + i] = (double)v[(size_t)g * d + i];
    }

  /* (3)+(4) Near field [P1 §2.1 eq. O_near] and dual-channel fusion
   * [P1 §2.1 eq. O]: x[h] = softmax(q_h K^T / sqrt(d)) V + alpha_far * S[g(h)]. */
  const long long j0 = (t - K + 1 > 0) ? t - K + 1 : 0;
  const int nwin = (int)(t - j0 + 1);
  const double scale = 1.0 / sqrt((double)d);
  for (int h = 0; h < nq; ++h) {
    const int g = h / group;
    const float* qh = q + (size_t)h * d;
    double m = -INFINITY;
    for (int a = 0; a < nwin; ++a) {
      const int slot = (int)((j0 + a) % K);
      const double* kj = &st->win_k[((size_t)slot * nkv + g) * d];
      double dot = 0.0;
      for (int i = 0; i < d; ++i) dot += (double)qh[i] * kj[i];
      s[a] = dot * scale;
      if (s[a] > m) m = s[a];
    }
    double denom = 0.0;
    for (int a = 0; a < nwin; ++a) {
      s[a] = exp(s[a] - m);
      denom += s[a];
    }
    for (int i = 0; i < d; ++i) {
      double o = 0.0;
      for (int a = 0; a < nwin; ++a) {
        const int slot = (int)((j0 + a) % K);
        o += s[a] * st->win_v[((size_t)slot * nkv + g) * d + i];
      }
      x[(size_t)h * d + i] = o / denom + p->alpha_far * st->S[(size_t)g * d + i];
    }
  }

  /* (5) Ring-buffer channel [P3 §2.1 channel 1, §2.4 kernel]: store x_t in
   * slot t mod ring_size, mean over all ring_size slots. */
  const int rslot = (int)(t % R);
  memcpy(&st->ring[(size_t)rslot * H], x, sizeof(double) * (size_t)H);

  /* (6) EMA field [P3 §2.1 channel 2]: field = gamma*field + (1-gamma)*x_t. */
  for (int i = 0; i < H; ++i)
    st->field[i] = p->ema_gamma * st->field[i] + (1.0 - p->ema_gamma) * x[i];

  /* (7) Semantic pool [P3 §2.1 channel 3]: weights softmax(cos(x, slot_j)/T),
   * semantic term = sum_j w_j slot_j. */
  double xx = 0.0;
  for (int i = 0; i < H; ++i) xx += x[i] * x[i];
  const double nx = fmax(sqrt(xx), SFA_ORACLE_NORM_FLOOR);
  double cmax = -INFINITY;
  for (int j = 0; j < P; ++j) {
    const float* sj = slots + (size_t)j * H;
    double dot = 0.0;
    for (int i = 0; i < H; ++i) dot += x[i] * (double)sj[i];
    c[j] = dot / (nx * fmax(slot_norm[j], SFA_ORACLE_NORM_FLOOR)) / p->temperature;
    if (c[j] > cmax) cmax = c[j];
  }
  double wsum = 0.0;
  for (int j = 0; j < P; ++j) {
    w[j] = exp(c[j] - cmax);
    wsum += w[j];
  }
  for (int j = 0; j < P; ++j) w[j] /= wsum;

  /* (8) Fusion, clip, layer scale, residual add [P3 §2.2]. */
  for (int i = 0; i < H; ++i) {
    double ring_mean = 0.0;
    for (int r = 0; r < R; ++r) ring_mean += st->ring[(size_t)r * H + i];
    ring_mean /= (double)R;
    double sem = 0.0;
    for (int j = 0; j < P; ++j) sem += w[j] * (double)slots[(size_t)j * H + i];
    double u = ring_mean + 0.5 * st->field[i] + 0.5 * sem;
    if (u > p->clip_eps) u = p->clip_eps;
    if (u < -p->clip_eps) u = -p->clip_eps;
    out[i] = x[i] + alpha_layer * u;
  }

  st->pos = t + 1;
}

int sfa_oracle_stream_run(const sfa_oracle_params* p, double alpha_layer,
                          const float* slots, const float* q, const float* k,
                          const float* v, long long n, sfa_oracle_stream* st,
                          double* out) {
  if (!params_ok(p) || !st || n < 0) return -1;
  if (n == 0) return 0;
  const int H = p->n_q_heads * p->head_dim;
  const int P = p->n_slots;
  double* slot_norm = (double*)malloc(sizeof(double) * (size_t)P);
  double* scratch = (double*)malloc(sizeof(double) * ((size_t)p->window_k + (size_t)H + 2u * (size_t)P));
  if (!slot_norm || !scratch) {
    free(slot_norm);
    free(scratch);
    return -1;
  }
  for (int j = 0; j < P; ++j) {
    double ss = 0.0;
    for (int i = 0; i < H; ++i) {
      const double e = (double)slots[(size_t)j * H + i];
      ss += e * e;
    }
    slot_norm[j] = sqrt(ss);
  }
  const size_t qs = (size_t)p->n_q_heads * p->head_dim;
  const size_t ks = (size_t)p->n_kv_heads * p->head_dim;
  for (long long t = 0; t < n; ++t)
    oracle_token(p, alpha_layer, slots, slot_norm, q + (size_t)t * qs, k + (size_t)t * ks,
                 v + (size_t)t * ks, st, out + (size_t)t * H, scratch);
  free(slot_norm);
  free(scratch);
  return 0;
}

int sfa_oracle_run_streams(const sfa_oracle_params* p, int n_streams,
                           const double* alpha_layer, const float* const* slots,
                           const float* const* q, const float* const* k,
                           const float* const* v, long long n,
                           sfa_oracle_stream* const* st, double* const* out,
                           int* threads_used) {
  if (!params_ok(p) || n_streams < 0 || n < 0) return -1;
  int bad = 0;
  int used = 1;
#ifdef _OPENMP
#pragma omp parallel reduction(| : bad)
  {
#pragma omp single
    used = omp_get_num_threads();
#pragma omp for schedule(dynamic, 1)
    for (int s = 0; s < n_streams; ++s)
      bad |= (sfa_oracle_stream_run(p, alpha_layer[s], slots[s], q[s], k[s], v[s], n, st[s],
                                    out[s]) != 0);
  }
#else
  for (int s = 0; s < n_streams; ++s)
    bad |= (sfa_oracle_stream_run(p, alpha_layer[s], slots[s], q[s], k[s], v[s], n, st[s],
                                  out[s]) != 0);
#endif
  if (threads_used) *threads_used = (n_streams < used) ? n_streams : used;
  return bad ? -1 : 0;
}
