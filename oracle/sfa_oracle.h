/*
 * sfa_oracle.h — plain fp64 CPU oracle of the Signal Field Attention operator.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * CPU-baseline leg of bench.py may load it.  The CUDA library never calls it
 * and shares no code with it.
 *
 * Sources (web pages):
 *   [P1] "Signal Field Attention (SFA)：8KB代码实现4.16倍推理加速与248倍内存压缩"
 *   [P2] "Signal Field Attention (SFA)" (project README page)
 *   [P3] "Dalin Soma SFA基于信号场注意力机制的神经网络推理加速框架"
 */
#ifndef SFA_ORACLE_H
#define SFA_ORACLE_H

#ifdef __cplusplus
extern "C" {
#endif

typedef struct sfa_oracle_params {
  int n_q_heads;
  int n_kv_heads;
  int head_dim;
  int window_k;      /* near-field window length k, [P1 §2.1] */
  int ring_size;     /* ring-buffer channel slots, [P3 §2.1 channel 1] */
  int n_slots;       /* semantic-pool slots, [P3 §2.1 channel 3] */
  double gamma_far;  /* far-field EWMA decay, [P1 §2.1 eq. S_t] */
  double alpha_far;  /* far-field mixing coefficient, [P1 §2.1 eq. O] */
  double ema_gamma;  /* EMA field decay, [P3 §2.1 channel 2] */
  double temperature;/* semantic-pool temperature, [P3 §2.1 channel 3] */
  double clip_eps;   /* enhancement clip, [P3 §2.2] */
} sfa_oracle_params;

/* State of one (layer, sequence) stream, all fp64, caller-owned arrays. */
typedef struct sfa_oracle_stream {
  double* win_k;  /* [window_k][n_kv_heads][head_dim], slot of position j is j mod k */
  double* win_v;  /* same layout */
  double* S;      /* [n_kv_heads][head_dim] far-field state */
  double* ring;   /* [ring_size][hidden], slot of position j is j mod ring_size */
  double* field;  /* [hidden] */
  long long pos;  /* number of tokens folded in so far */
} sfa_oracle_stream;

/* alpha_layer = alpha_base * (0.3 + 0.7 * layer/(L-1)) * cross_decay^layer;
 * layer/(L-1) is taken as 0 when L == 1.  [P3 §2.2], [P2 cross-layer decay formula] */
double sfa_oracle_alpha_layer(double alpha_base, double cross_decay, int layer, int n_layers);

/* Runs n tokens of one stream, token by token.
 *   slots: [n_slots][hidden] (fp32 storage, read as exact values)
 *   q:     [n][n_q_heads][head_dim]; k, v: [n][n_kv_heads][head_dim]
 *          (fp32 storage; bf16 inputs are passed widened, which is exact)
 *   out:   [n][hidden] fp64
 * Returns 0, or -1 on invalid parameters. */
int sfa_oracle_stream_run(const sfa_oracle_params* p, double alpha_layer,
                          const float* slots, const float* q, const float* k,
                          const float* v, long long n, sfa_oracle_stream* st,
                          double* out);

/* Runs n tokens for n_streams independent streams (OpenMP over streams).
 * Arrays of per-stream pointers; *threads_used receives the thread count. */
int sfa_oracle_run_streams(const sfa_oracle_params* p, int n_streams,
                           const double* alpha_layer, const float* const* slots,
                           const float* const* q, const float* const* k,
                           const float* const* v, long long n,
                           sfa_oracle_stream* const* st, double* const* out,
                           int* threads_used);

#ifdef __cplusplus
}
#endif
#endif
