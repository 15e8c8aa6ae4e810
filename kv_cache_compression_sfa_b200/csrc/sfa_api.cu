// sfa_api.cu — the C ABI declared in include/sfa.h: configuration checks,
// state and workspace layout, handle set-up, launch configuration and the
// device error latch.
//
// Sources (web pages):
//   [P1] "Signal Field Attention (SFA)：8KB代码实现4.16倍推理加速与248倍内存压缩"
//   [P2] "Signal Field Attention (SFA)" (project README page): SFA_Config
//        defaults, engine init(n_layers, hidden) / per-layer enhancement call.
//   [P3] "Dalin Soma SFA基于信号场注意力机制的神经网络推理加速框架" §2.2:
//        alpha_layer = alpha_base·(0.3 + 0.7·layer_ratio)·decay^layer.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <algorithm>
#include <type_traits>
#include <cstring>
#include <new>
#include <vector>

#include "sfa_internal.h"

using namespace sfa;

struct sfa_handle {
  uint32_t magic;
  sfa_config cfg;        // cfg.slots points at the handle's own copy
  int device;
  float* slots;          // [L][64][H]
  float* slot_norm;      // [L][64]
  float* alpha_layer;    // [L]
  unsigned char* slot_img;  // [L][H/64][hi, lo] bf16 blocks for the prefill pool MMAs
  float* slot_dec;       // [L][cs][64][HS + 4] each decode CTA's slot slice, rows padded
  int* err;              // device error word
  uint64_t cfg_hash;
  int cs;               // CTAs per cluster of the decode kernels
  int n_sm;              // streaming multiprocessors of the device
  NearPlan near;         // shared-memory plan of the prefill near-field kernel
  NearPlan near_small;   // near_mode 3: the plan for calls below kFusedMinTilesPerSm tiles per SM
  int decode_budget;
  unsigned spin_limit;
  long long withhold_tile;
  bool tile_ok;          // the batch-tiled decode fits this configuration
  TilePlan tile_plan;    // its shared-memory plan
  int tile_mode;         // -1: by batch size; 0: never; 1: always (sfa_debug_set_paths)
  int near_mode;         // prefill near field where the tensor cores apply: 3 by call size (2
                         // for large calls, else 1), 2 fused with the pool scores, 1 tensor
                         // cores and a separate pool kernel, 0 CUDA cores
  bool inputs_early;     // decode inputs declared complete before each call
  int out_mode;          // sfa_out_mode of the compute calls
};

namespace {

constexpr uint32_t kHandleMagic = 0x48414653u;  // "SFAH"
constexpr long long kBlkBytesHost = 64 * 64 * 2;  // one 64 x 64 bf16 block

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int hidden_of(const sfa_config* c) { return c->n_q_heads * c->head_dim; }

size_t in_bytes(int dtype) { return dtype == SFA_F32 ? 4 : 2; }

uint64_t fnv1a(uint64_t h, const void* data, size_t n) {
  const unsigned char* p = static_cast<const unsigned char*>(data);
  for (size_t i = 0; i < n; ++i) {
    h ^= p[i];
    h *= 1099511628211ull;
  }
  return h;
}

uint64_t config_hash(const sfa_config* c) {
  uint64_t h = 1469598103934665603ull;
  const int ints[] = {c->n_layers, c->n_q_heads, c->n_kv_heads, c->head_dim, c->window_k,
                      c->ring_size, c->n_slots, c->in_dtype, SFA_ABI_VERSION};
  const float flts[] = {c->gamma_far, c->alpha_far, c->ema_gamma, c->temperature,
                        c->clip_eps, c->alpha_base, c->cross_decay};
  h = fnv1a(h, ints, sizeof(ints));
  h = fnv1a(h, flts, sizeof(flts));
  return h;
}

StreamOffsets stream_offsets(const sfa_config* c) {
  const long long H = hidden_of(c);
  const long long win = static_cast<long long>(c->window_k) * c->n_kv_heads * c->head_dim *
                        static_cast<long long>(in_bytes(c->in_dtype));
  StreamOffsets o;
  o.pos = 0;
  o.win_k = 256;
  o.win_v = o.win_k + align256(win);
  o.far = o.win_v + align256(win);
  o.field = o.far + align256(4LL * c->n_kv_heads * c->head_dim);
  o.ring_sum = o.field + align256(4 * H);
  o.ring = o.ring_sum + align256(4 * H);
  o.stride = o.ring + align256(4LL * kRing * H);
  return o;
}

// Smallest cluster whose per-CTA hidden slice is at most `max_slice`.
int smallest_cluster(int nq, int d, int max_slice) {
  for (int cs = 1; cs <= kMaxCluster; ++cs)
    if (nq % cs == 0 && (nq / cs) * d <= max_slice) return cs;
  return 0;
}

// Cluster sizes to try, best first: slices of at most 256 hidden elements
// (smallest cluster first), then at most 512.
std::vector<int> cluster_candidates(int nq, int d) {
  std::vector<int> out;
  for (int lim : {256, kMaxSlice})
    for (int cs = 1; cs <= kMaxCluster; ++cs)
      if (nq % cs == 0 && (nq / cs) * d <= lim &&
          std::find(out.begin(), out.end(), cs) == out.end())
        out.push_back(cs);
  return out;
}

// Workspace of a prefill call: the streams' positions, S at the end of the
// call, the pool weights of every tile (two 8 KB bf16 blocks) and S at
// every tile start.
// Segments of the output kernel's tile walk: about four rounds of two CTAs
// per SM over (stream, 64-column block, segment).
int out_segments(int n_sm, int hidden, long long streams, long long tiles_per_stream) {
  const long long units = streams * (hidden / 64);
  const long long target = 4LL * 2 * std::max(n_sm, 1);
  long long nseg = std::max(1LL, std::min(tiles_per_stream, (target + units - 1) / units));
  const long long tps = (tiles_per_stream + nseg - 1) / nseg;
  return static_cast<int>((tiles_per_stream + tps - 1) / tps);
}

PrefillWorkspace prefill_workspace(const sfa_config* c, int layers, int batch, long long n, int out_mode,
                                   int n_sm) {
  PrefillWorkspace w;
  const long long streams = static_cast<long long>(layers) * batch;
  const long long tps = (n + kTile - 1) / kTile;
  const long long tiles = streams * tps;
  const long long sdim = static_cast<long long>(c->n_kv_heads) * c->head_dim;
  const long long H = hidden_of(c);
  w.pos = 0;
  w.sfin = align256(8 * streams);
  w.w = w.sfin + align256(4 * streams * sdim);
  w.sst = w.w + tiles * 2LL * kBlkBytesHost;
  w.x = w.sst + align256(4 * tiles * sdim);
  // x between the kernels, where the result buffer cannot hold it
  const long long xb = out_mode == SFA_OUT_F32 ? 0 : align256(4LL * streams * n * H);
  w.fagg = w.x + xb;
  w.halo = w.fagg + align256(4LL * tiles * H);
  w.total = w.halo + align256(4LL * streams * out_segments(n_sm, static_cast<int>(H), streams, tps) * kHalo * H);
  return w;
}

// Limits of one prefill call: its kernels put the layers x batch streams in
// gridDim.y (at most 65535) and count a stream's tiles in 32 bits.  Checked
// before any size arithmetic, which these bounds keep below 2^63.
int prefill_shape_status(int layers, int batch, long long n) {
  if (static_cast<long long>(layers) * batch > 65535) return SFA_ERR_UNSUPPORTED;
  if (n > 0x7fffffffLL * kTile) return SFA_ERR_UNSUPPORTED;
  return SFA_OK;
}

// Most KV heads any CTA of a cluster of `cs` needs.
int max_kv_heads_per_cta(int nq, int nkv, int cs) {
  const int hpc = nq / cs, g = nq / nkv;
  int best = 0;
  for (int r = 0; r < cs; ++r) {
    const int h0 = r * hpc;
    best = std::max(best, (h0 + hpc - 1) / g - h0 / g + 1);
  }
  return best;
}

int decode_budget(size_t limit) {
  return static_cast<int>(std::min(static_cast<size_t>(kDecodeSmemBudget), limit));
}

bool handle_ok(const sfa_handle* h) { return h != nullptr && h->magic == kHandleMagic; }

int cuda_status(cudaError_t e) { return e == cudaSuccess ? SFA_OK : SFA_ERR_CUDA; }

// Near-field plan of the prefill: on the tensor cores where they apply (bf16
// inputs, k <= 16) unless h->near_mode is 0, there fused with the pool
// scores unless it is 1; else on the CUDA cores.
bool plan_near_field(sfa_handle* h, size_t limit) {
  const sfa_config* c = &h->cfg;
  const int esz = static_cast<int>(in_bytes(c->in_dtype));
  const bool fused = h->near_mode >= 2;
  if (!((h->near_mode > 0 && plan_near(c->head_dim, esz, c->window_k, limit, true, fused, &h->near)) ||
        plan_near(c->head_dim, esz, c->window_k, limit, false, false, &h->near)))
    return false;
  h->near_small = h->near;
  if (h->near_mode == 3 && h->near.fused &&
      !plan_near(c->head_dim, esz, c->window_k, limit, true, false, &h->near_small))
    h->near_small = h->near;
  return true;
}

template <typename P>
void fill_common(P& p, const sfa_handle* h, int batch, void* state) {
  const sfa_config* c = &h->cfg;
  p.state = static_cast<unsigned char*>(state);
  p.slots = h->slots;
  p.slot_norm = h->slot_norm;
  p.slot_img = h->slot_img;
  if constexpr (std::is_same<P, DecodeParams>::value) p.slot_dec = h->slot_dec;
  p.alpha_layer = h->alpha_layer;
  p.err = h->err;
  p.cfg_hash = h->cfg_hash;
  p.so = stream_offsets(c);
  p.L = c->n_layers;
  p.B = batch;
  p.nq = c->n_q_heads;
  p.nkv = c->n_kv_heads;
  p.K = c->window_k;
  p.H = hidden_of(c);
  p.G = c->n_q_heads / c->n_kv_heads;
  p.gamma_far = c->gamma_far;
  p.alpha_far = c->alpha_far;
  p.ema_gamma = c->ema_gamma;
  p.inv_temp = 1.0f / c->temperature;
  p.clip_eps = c->clip_eps;
  p.score_scale = static_cast<float>(1.0 / std::sqrt(static_cast<double>(c->head_dim)));
}

int prefill_impl(const sfa_handle* h, int layer_begin, int layer_count, const void* q, const void* k,
                 const void* v, long long n, const int* lens, int batch, void* state, void* out,
                 void* workspace, size_t workspace_bytes, void* stream);

}  // namespace

extern "C" {

void sfa_config_default(sfa_config* c) {
  if (!c) return;
  std::memset(c, 0, sizeof(*c));
  c->window_k = 16;
  c->gamma_far = 0.9f;
  c->alpha_far = 0.1f;
  c->ring_size = kRing;
  c->ema_gamma = 0.98f;
  c->n_slots = kSlots;
  c->temperature = 0.07f;
  c->clip_eps = 0.5f;
  c->alpha_base = 0.1f;
  c->cross_decay = 0.8f;
  c->in_dtype = SFA_BF16;
  c->slots = nullptr;
}

int sfa_config_validate(const sfa_config* c) {
  if (!c) return SFA_ERR_INVALID_ARG;
  if (c->n_layers <= 0 || c->n_q_heads <= 0 || c->n_kv_heads <= 0 || c->head_dim <= 0 ||
      c->window_k <= 0 || c->ring_size <= 0 || c->n_slots <= 0)
    return SFA_ERR_INVALID_ARG;
  if (c->n_q_heads % c->n_kv_heads != 0) return SFA_ERR_INVALID_ARG;
  const float scalars[] = {c->gamma_far, c->alpha_far, c->ema_gamma, c->temperature,
                           c->clip_eps, c->alpha_base, c->cross_decay};
  for (float s : scalars)
    if (!std::isfinite(s)) return SFA_ERR_INVALID_ARG;
  if (c->gamma_far < 0.f || c->gamma_far > 1.f || c->ema_gamma < 0.f || c->ema_gamma > 1.f)
    return SFA_ERR_INVALID_ARG;
  if (!(c->temperature > 0.f) || !std::isfinite(1.0f / c->temperature) || c->clip_eps < 0.f)
    return SFA_ERR_INVALID_ARG;
  if (c->in_dtype != SFA_F32 && c->in_dtype != SFA_BF16) return SFA_ERR_INVALID_ARG;
  if (c->slots == nullptr) return SFA_ERR_INVALID_ARG;
  if (!aligned16(c->slots)) return SFA_ERR_ALIGNMENT;
  if (c->head_dim != 64 && c->head_dim != 128) return SFA_ERR_UNSUPPORTED;
  if (c->window_k > kMaxWindow || c->ring_size != kRing || c->n_slots != kSlots)
    return SFA_ERR_UNSUPPORTED;
  if (static_cast<long long>(c->n_q_heads) * c->head_dim > kMaxHidden) return SFA_ERR_UNSUPPORTED;
  if (smallest_cluster(c->n_q_heads, c->head_dim, kMaxSlice) == 0) return SFA_ERR_UNSUPPORTED;
  return SFA_OK;
}

int sfa_state_layout_for(const sfa_config* c, int batch, sfa_state_layout* out) {
  if (!c || !out || batch <= 0) return SFA_ERR_INVALID_ARG;
  const int v = sfa_config_validate(c);
  if (v != SFA_OK) return v;
  const StreamOffsets o = stream_offsets(c);
  out->header_bytes = kHeaderBytes;
  out->stream_stride = static_cast<size_t>(o.stride);
  out->total_bytes = kHeaderBytes + static_cast<size_t>(o.stride) * c->n_layers * batch;
  out->off_pos = static_cast<size_t>(o.pos);
  out->off_win_k = static_cast<size_t>(o.win_k);
  out->off_win_v = static_cast<size_t>(o.win_v);
  out->off_far = static_cast<size_t>(o.far);
  out->off_field = static_cast<size_t>(o.field);
  out->off_ring_sum = static_cast<size_t>(o.ring_sum);
  out->off_ring = static_cast<size_t>(o.ring);
  return SFA_OK;
}

int sfa_init(const sfa_config* cfg, sfa_handle** out) {
  if (!out) return SFA_ERR_INVALID_ARG;
  *out = nullptr;
  const int v = sfa_config_validate(cfg);
  if (v != SFA_OK) return v;
  sfa_handle* h = new (std::nothrow) sfa_handle();
  if (!h) return SFA_ERR_CUDA;
  h->magic = kHandleMagic;
  h->cfg = *cfg;
  h->cfg_hash = config_hash(cfg);
  h->cs = 0;
  h->spin_limit = kDefaultSpinLimit;
  h->withhold_tile = -1;
  h->inputs_early = false;
  h->tile_mode = -1;
  h->near_mode = 3;
  h->out_mode = SFA_OUT_F32;
  const int L = cfg->n_layers, H = hidden_of(cfg);
  bool no_fit = false;  // a kernel's shared-memory plan does not fit this device
  const size_t slot_bytes = sizeof(float) * static_cast<size_t>(L) * kSlots * H;
  cudaError_t e = cudaGetDevice(&h->device);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&h->n_sm, cudaDevAttrMultiProcessorCount, h->device);
  if (e == cudaSuccess) e = cudaMalloc(&h->slots, slot_bytes);
  if (e == cudaSuccess) e = cudaMalloc(&h->slot_norm, sizeof(float) * L * kSlots);
  if (e == cudaSuccess) e = cudaMalloc(&h->alpha_layer, sizeof(float) * L);
  if (e == cudaSuccess) e = cudaMalloc(&h->err, sizeof(int));
  if (e == cudaSuccess) e = cudaMalloc(&h->slot_img, slot_bytes);  // bf16 hi + lo per slot element
  if (e == cudaSuccess) e = cudaMemcpy(h->slots, cfg->slots, slot_bytes, cudaMemcpyDefault);
  if (e == cudaSuccess) e = cudaMemset(h->err, 0, sizeof(int));
  if (e == cudaSuccess) e = prefill_prepare(h->device);
  if (e == cudaSuccess) e = decode_prepare(h->device);
  if (e == cudaSuccess) e = decode_tile_prepare(h->device);
  if (e == cudaSuccess) {
    // Prefill near-field plan; the decode kernels' cluster size: the first
    // candidate whose decode plan fits and of which one cluster fits on the
    // device.
    const size_t limit = prefill_smem_limit(h->device);
    const int esz = static_cast<int>(in_bytes(cfg->in_dtype));
    if (!plan_near_field(h, limit)) no_fit = true;
    if (static_cast<size_t>(std::max(prefill_pool_smem(), prefill_out_smem())) > limit)
      no_fit = true;
    if (no_fit) e = cudaErrorInvalidConfiguration;
    for (int cs : cluster_candidates(cfg->n_q_heads, cfg->head_dim)) {
      if (e != cudaSuccess) break;
      const int hpc = cfg->n_q_heads / cs;
      const size_t dsm = decode_smem_bytes(hpc, cfg->head_dim, esz,
                                           max_kv_heads_per_cta(cfg->n_q_heads, cfg->n_kv_heads, cs),
                                           cfg->n_kv_heads, cfg->window_k, decode_budget(limit));
      if (dsm > limit) continue;
      if (decode_max_active_clusters(cs, dsm, cfg->in_dtype, cfg->head_dim) < 1) continue;
      h->cs = cs;
      h->decode_budget = decode_budget(limit);
      h->tile_ok = plan_decode_tile(hidden_of(cfg), cfg->head_dim, esz, cfg->n_q_heads / cfg->n_kv_heads,
                                    cfg->window_k, limit, &h->tile_plan);
      break;
    }
    if (e == cudaSuccess && h->cs == 0) {
      no_fit = true;
      e = cudaErrorInvalidConfiguration;
    }
    if (e == cudaSuccess) {
      // Each decode CTA's slot slice [64][HS] laid out contiguously with the
      // rows padded to HS + 4 floats, as in its shared memory: one bulk copy.
      const int hs = (cfg->n_q_heads / h->cs) * cfg->head_dim;
      const size_t pitch = static_cast<size_t>(hs + 4) * sizeof(float);
      const size_t bytes = static_cast<size_t>(L) * h->cs * kSlots * pitch;
      e = cudaMalloc(&h->slot_dec, bytes);
      if (e == cudaSuccess) e = cudaMemset(h->slot_dec, 0, bytes);
      for (int l = 0; l < L && e == cudaSuccess; ++l)
        for (int r = 0; r < h->cs && e == cudaSuccess; ++r)
          e = cudaMemcpy2D(h->slot_dec + (static_cast<size_t>(l) * h->cs + r) * kSlots * (hs + 4), pitch,
                           h->slots + static_cast<size_t>(l) * kSlots * H + static_cast<size_t>(r) * hs,
                           sizeof(float) * H, sizeof(float) * hs, kSlots, cudaMemcpyDeviceToDevice);
    }
  }
  if (e == cudaSuccess) e = launch_slot_norms(h->slots, h->slot_norm, L, H, nullptr);
  if (e == cudaSuccess) e = launch_slot_image(h->slots, h->slot_img, L, H, nullptr);
  if (e == cudaSuccess) {
    // [P3 §2.2] alpha_layer = alpha_base*(0.3 + 0.7*layer/(L-1))*decay^layer;
    // the ratio is 0 for a single-layer model.
    std::vector<float> a(L);
    for (int l = 0; l < L; ++l) {
      const double ratio = L > 1 ? static_cast<double>(l) / (L - 1) : 0.0;
      a[l] = static_cast<float>(static_cast<double>(cfg->alpha_base) * (0.3 + 0.7 * ratio) *
                                std::pow(static_cast<double>(cfg->cross_decay), l));
    }
    e = cudaMemcpy(h->alpha_layer, a.data(), sizeof(float) * L, cudaMemcpyHostToDevice);
  }
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e != cudaSuccess) {
    cudaGetLastError();
    cudaFree(h->slots);
    cudaFree(h->slot_norm);
    cudaFree(h->alpha_layer);
    cudaFree(h->slot_img);
    cudaFree(h->slot_dec);
    cudaFree(h->err);
    h->magic = 0;
    delete h;
    return no_fit ? SFA_ERR_UNSUPPORTED : SFA_ERR_CUDA;
  }
  h->cfg.slots = h->slots;
  *out = h;
  return SFA_OK;
}

int sfa_destroy(sfa_handle* h) {
  if (!handle_ok(h)) return SFA_ERR_INVALID_ARG;
  cudaError_t e = cudaDeviceSynchronize();
  cudaFree(h->slots);
  cudaFree(h->slot_norm);
  cudaFree(h->alpha_layer);
  cudaFree(h->slot_img);
  cudaFree(h->slot_dec);
  cudaFree(h->err);
  h->magic = 0;
  delete h;
  return cuda_status(e);
}

size_t sfa_state_bytes(const sfa_handle* h, int batch) {
  if (!handle_ok(h) || batch <= 0) return 0;
  sfa_state_layout lay;
  if (sfa_state_layout_for(&h->cfg, batch, &lay) != SFA_OK) return 0;
  return lay.total_bytes;
}

size_t sfa_prefill_workspace_bytes(const sfa_handle* h, int batch, long long n) {
  if (!handle_ok(h)) return 0;
  return sfa_prefill_layers_workspace_bytes(h, h->cfg.n_layers, batch, n);
}

size_t sfa_prefill_layers_workspace_bytes(const sfa_handle* h, int layer_count, int batch,
                                          long long n) {
  if (!handle_ok(h) || batch <= 0 || n <= 0 || layer_count <= 0 ||
      layer_count > h->cfg.n_layers)
    return 0;
  if (prefill_shape_status(layer_count, batch, n) != SFA_OK) return 0;
  return static_cast<size_t>(prefill_workspace(&h->cfg, layer_count, batch, n, h->out_mode, h->n_sm).total);
}

int sfa_state_reset(const sfa_handle* h, void* state, int batch, void* stream) {
  if (!handle_ok(h) || !state || batch <= 0) return SFA_ERR_INVALID_ARG;
  if (!aligned16(state)) return SFA_ERR_ALIGNMENT;
  const size_t bytes = sfa_state_bytes(h, batch);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(state, 0, bytes, s);
  if (e != cudaSuccess) return SFA_ERR_CUDA;
  StateHeader hd;
  std::memset(&hd, 0, sizeof(hd));
  hd.magic = kMagic;
  hd.abi = SFA_ABI_VERSION;
  hd.cfg_hash = h->cfg_hash;
  hd.batch = batch;
  hd.n_layers = h->cfg.n_layers;
  hd.stream_stride = static_cast<uint64_t>(stream_offsets(&h->cfg).stride);
  return cuda_status(launch_write_header(static_cast<unsigned char*>(state), hd, s));
}

int sfa_prefill(const sfa_handle* h, const void* q, const void* k, const void* v, long long n,
                int batch, void* state, void* out, void* workspace, size_t workspace_bytes,
                void* stream) {
  if (!handle_ok(h)) return SFA_ERR_INVALID_ARG;
  return sfa_prefill_layers(h, 0, h->cfg.n_layers, q, k, v, n, batch, state, out, workspace,
                            workspace_bytes, stream);
}

int sfa_prefill_layers(const sfa_handle* h, int layer_begin, int layer_count, const void* q,
                       const void* k, const void* v, long long n, int batch, void* state,
                       void* out, void* workspace, size_t workspace_bytes, void* stream) {
  return prefill_impl(h, layer_begin, layer_count, q, k, v, n, nullptr, batch, state, out, workspace,
                      workspace_bytes, stream);
}

int sfa_prefill_ragged(const sfa_handle* h, const void* q, const void* k, const void* v, long long n_max,
                       const int* lens, int batch, void* state, void* out, void* workspace,
                       size_t workspace_bytes, void* stream) {
  if (!handle_ok(h) || !lens) return SFA_ERR_INVALID_ARG;
  return prefill_impl(h, 0, h->cfg.n_layers, q, k, v, n_max, lens, batch, state, out, workspace,
                      workspace_bytes, stream);
}

}  // extern "C"

namespace {

int prefill_impl(const sfa_handle* h, int layer_begin, int layer_count, const void* q, const void* k,
                 const void* v, long long n, const int* lens, int batch, void* state, void* out,
                 void* workspace, size_t workspace_bytes, void* stream) {
  if (!handle_ok(h) || n < 0 || batch <= 0) return SFA_ERR_INVALID_ARG;
  if (layer_begin < 0 || layer_count <= 0 || layer_begin + layer_count > h->cfg.n_layers)
    return SFA_ERR_INVALID_ARG;
  if (n == 0) return SFA_OK;
  if (!q || !k || !v || !state || !out) return SFA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(state) || !aligned16(out) ||
      !aligned16(workspace))
    return SFA_ERR_ALIGNMENT;
  const int shape = prefill_shape_status(layer_count, batch, n);
  if (shape != SFA_OK) return shape;
  const sfa_config* c = &h->cfg;
  const PrefillWorkspace w = prefill_workspace(c, layer_count, batch, n, h->out_mode, h->n_sm);
  if (!workspace || workspace_bytes < static_cast<size_t>(w.total)) return SFA_ERR_WORKSPACE;
  const long long streams = static_cast<long long>(layer_count) * batch;
  const long long tiles_per_stream = (n + kTile - 1) / kTile;
  // the tensor copies of the near field address token rows with 32-bit coordinates
  if (h->near.tc && streams * n > 0x7fffffffLL) return SFA_ERR_UNSUPPORTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  PrefillParams p;
  std::memset(&p, 0, sizeof(p));
  fill_common(p, h, batch, state);
  p.q = q;
  p.k = k;
  p.v = v;
  p.ws = static_cast<unsigned char*>(workspace);
  p.res = out;
  p.out_mode = h->out_mode;
  // x between the kernels: in the result buffer itself (fp32 x + enhancement
  // overwrites it row by row) or in the workspace
  p.out = h->out_mode == SFA_OUT_F32 ? static_cast<float*>(out) : reinterpret_cast<float*>(p.ws + w.x);
  p.n = n;
  p.lens = lens;
  p.l0 = layer_begin;
  p.tiles_per_stream = static_cast<int>(tiles_per_stream);
  p.n_streams = static_cast<int>(streams);
  p.ws_pos = w.pos;
  p.ws_sfin = w.sfin;
  p.ws_w = w.w;
  p.ws_sst = w.sst;
  p.ws_x = w.x;
  p.ws_fagg = w.fagg;
  p.ws_halo = w.halo;
  p.nseg_out = out_segments(h->n_sm, hidden_of(c), streams, tiles_per_stream);
  p.tps_out = static_cast<int>((tiles_per_stream + p.nseg_out - 1) / p.nseg_out);
  // Calls of few tiles per SM leave the fused kernel (one CTA per SM walking
  // every head) with too little to overlap: they take the two-kernel path.
  const NearPlan& np = (h->near_mode == 3 && streams * tiles_per_stream < kFusedMinTilesPerSm * h->n_sm)
                           ? h->near_small : h->near;
  if (np.fused) {
    // Fused kernel: one CTA per SM, each a run of consecutive tiles of one
    // stream, all heads; about one round over the SMs.
    const long long total = streams * tiles_per_stream;
    const long long tps = std::min(tiles_per_stream, std::max(1LL, (total + h->n_sm - 1) / std::max(h->n_sm, 1)));
    const long long nseg = (tiles_per_stream + tps - 1) / tps;
    p.n_seg = static_cast<int>(nseg);
    p.tps = static_cast<int>(tps);
  } else {
    // Near-field segments: about four rounds of two CTAs per SM, each CTA a
    // run of consecutive tiles of one (stream, head).
    const long long units = static_cast<long long>(c->n_q_heads) * streams;
    const long long target = 4LL * 2 * std::max(h->n_sm, 1);
    long long nseg = std::max(1LL, std::min(tiles_per_stream, (target + units - 1) / units));
    const long long tps = (tiles_per_stream + nseg - 1) / nseg;
    nseg = (tiles_per_stream + tps - 1) / tps;
    if (nseg * c->n_q_heads > 0x7fffffffLL) return SFA_ERR_UNSUPPORTED;
    p.n_seg = static_cast<int>(nseg);
    p.tps = static_cast<int>(tps);
  }
  p.spin_limit = h->spin_limit;
  p.withhold_tile = h->withhold_tile;
  p.near = np;
  p.pool_smem = prefill_pool_smem();
  p.out_smem = prefill_out_smem();
  return cuda_status(launch_prefill(p, c->in_dtype, c->head_dim, s));
}

}  // namespace

extern "C" {

int sfa_decode_step(const sfa_handle* h, const void* q, const void* k, const void* v, int batch,
                    void* state, void* out, void* stream) {
  if (!handle_ok(h)) return SFA_ERR_INVALID_ARG;
  return sfa_decode_step_ex(h, 0, h->cfg.n_layers, nullptr, batch, q, k, v, batch, state, out,
                            stream);
}

int sfa_decode_step_ex(const sfa_handle* h, int layer_begin, int layer_count, const int* seq_ids,
                       int n_seq, const void* q, const void* k, const void* v, int batch,
                       void* state, void* out, void* stream) {
  if (!handle_ok(h) || batch <= 0 || !q || !k || !v || !state || !out) return SFA_ERR_INVALID_ARG;
  if (layer_begin < 0 || layer_count <= 0 || layer_begin + layer_count > h->cfg.n_layers)
    return SFA_ERR_INVALID_ARG;
  if (n_seq <= 0 || (seq_ids == nullptr && n_seq != batch) || n_seq > batch)
    return SFA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(state) || !aligned16(out))
    return SFA_ERR_ALIGNMENT;
  const sfa_config* c = &h->cfg;
  if (n_seq > 65535 || layer_count > 65535) return SFA_ERR_UNSUPPORTED;
  DecodeParams p;
  std::memset(&p, 0, sizeof(p));
  fill_common(p, h, batch, state);
  p.l0 = layer_begin;
  p.Lc = layer_count;
  p.seq_ids = seq_ids;
  p.n_seq = n_seq;
  p.q = q;
  p.k = k;
  p.v = v;
  p.out = static_cast<float*>(out);  // the batch-tiled decode keeps x here (SFA_OUT_F32 only)
  p.res = out;
  p.out_mode = h->out_mode;
  p.CS = h->cs;
  p.HPC = c->n_q_heads / p.CS;
  p.NGm = max_kv_heads_per_cta(c->n_q_heads, c->n_kv_heads, p.CS);
  p.smem_budget = h->decode_budget;
  p.tp = h->tile_plan;
  p.inputs_early = h->inputs_early ? 1 : 0;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // Batch-tiled decode from kDecodeTileMinSeqs sequences per call (its
  // tensor copies address input rows with 32-bit coordinates; it keeps x in
  // out, so only for fp32 x + enhancement results).
  const bool tile = h->tile_ok && static_cast<long long>(layer_count) * n_seq <= 0x7fffffffLL &&
                    h->out_mode == SFA_OUT_F32 &&
                    (h->tile_mode == 1 || (h->tile_mode < 0 && n_seq >= kDecodeTileMinSeqs));
  if (tile) return cuda_status(launch_decode_tile(p, c->in_dtype, c->head_dim, s));
  return cuda_status(launch_decode(p, c->in_dtype, c->head_dim, s));
}

int sfa_check_device_status(const sfa_handle* h, void* stream) {
  if (!handle_ok(h)) return SFA_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return SFA_ERR_CUDA;
  int code = 0;
  e = cudaMemcpy(&code, h->err, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return SFA_ERR_CUDA;
  if (code != 0) {
    e = cudaMemset(h->err, 0, sizeof(int));
    if (e != cudaSuccess) return SFA_ERR_CUDA;
  }
  return code;
}

const char* sfa_status_string(int status) {
  switch (status) {
    case SFA_OK: return "ok";
    case SFA_ERR_INVALID_ARG: return "invalid argument";
    case SFA_ERR_UNSUPPORTED: return "unsupported configuration";
    case SFA_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
    case SFA_ERR_STATE_MISMATCH: return "state header does not match the handle or batch";
    case SFA_ERR_CUDA: return "CUDA error";
    case SFA_ERR_DEVICE_TIMEOUT: return "bounded device wait ran out";
    case SFA_ERR_WORKSPACE: return "workspace too small";
    default: return "unknown status";
  }
}

int sfa_abi_version(void) { return SFA_ABI_VERSION; }

int sfa_set_output_mode(sfa_handle* h, int mode) {
  if (!handle_ok(h) || mode < SFA_OUT_F32 || mode > SFA_OUT_ADD_BF16) return SFA_ERR_INVALID_ARG;
  h->out_mode = mode;
  return SFA_OK;
}

int sfa_set_decode_input_prefetch(sfa_handle* h, int enable) {
  if (!handle_ok(h) || (enable != 0 && enable != 1)) return SFA_ERR_INVALID_ARG;
  h->inputs_early = enable == 1;
  return SFA_OK;
}

int sfa_debug_set_wait_limit(sfa_handle* h, unsigned int spin_limit, long long withhold_tile) {
  if (!handle_ok(h)) return SFA_ERR_INVALID_ARG;
  h->spin_limit = spin_limit ? spin_limit : kDefaultSpinLimit;
  h->withhold_tile = withhold_tile < 0 ? -1 : withhold_tile;
  return SFA_OK;
}

int sfa_debug_set_paths(sfa_handle* h, int decode_tile, int prefill_near) {
  if (!handle_ok(h) || decode_tile < -1 || decode_tile > 1 || prefill_near < 0 || prefill_near > 3)
    return SFA_ERR_INVALID_ARG;
  if (decode_tile == 1 && !h->tile_ok) return SFA_ERR_UNSUPPORTED;
  const int old_mode = h->near_mode;
  const NearPlan old_plan = h->near, old_small = h->near_small;
  h->near_mode = prefill_near;
  if (!plan_near_field(h, prefill_smem_limit(h->device))) {
    h->near_mode = old_mode;
    h->near = old_plan;
    h->near_small = old_small;
    return SFA_ERR_UNSUPPORTED;
  }
  h->tile_mode = decode_tile;
  return SFA_OK;
}

}  // extern "C"
