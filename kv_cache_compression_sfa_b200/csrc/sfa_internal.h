// sfa_internal.h — layouts and kernel parameter blocks shared by the host
// launch layer (sfa_api.cu) and the kernels (sfa_decode.cu, sfa_prefill.cu).
//
// Sources (web pages):
//   [P1] "Signal Field Attention (SFA)：8KB代码实现4.16倍推理加速与248倍内存压缩"
//   [P2] "Signal Field Attention (SFA)" (project README page)
//   [P3] "Dalin Soma SFA基于信号场注意力机制的神经网络推理加速框架"
#pragma once

#include <cuda_runtime.h>
#include <cstddef>
#include <cstdint>

#include "sfa.h"

namespace sfa {

constexpr uint32_t kMagic = 0x31414653u;  // "SFA1"
constexpr size_t kHeaderBytes = 256;
constexpr int kRing = 16;                 // ring-buffer slots [P3 §2.1 channel 1]
constexpr int kSlots = 64;                // semantic slots [P3 §2.1 channel 3]
constexpr int kMaxHidden = 8192;
constexpr int kMaxWindow = 256;
constexpr int kMaxSlice = 512;            // hidden elements owned by one CTA
constexpr int kMaxCluster = 16;           // largest (non-portable) cluster size
constexpr float kNormFloor = 1e-12f;      // cosine norm clamp

// Prefill tiling.
constexpr int kTile = 64;                 // tokens per prefill tile
constexpr int kHalo = kRing - 1;          // x rows a tile needs from before it
constexpr int kPrefillThreads = 256;
constexpr int kDecodeThreads = 256;
constexpr int kDecodeTileThreads = 256;     // batch-tiled decode (64 sequences per tile)
constexpr int kDecodeTileMinSeqs = 64;      // batch-tiled decode from this many sequences per call
constexpr int kDecodeTileMaxWindow = 64;    // ... and windows of at most this many positions
constexpr int kGroup = 16;                // tiles per look-back group

// Look-back flag values.
constexpr unsigned kFlagEmpty = 0u;
constexpr unsigned kFlagAgg = 1u;
constexpr unsigned kFlagIncl = 2u;
constexpr unsigned kDefaultSpinLimit = 1u << 21;

// First bytes of every state buffer.
struct StateHeader {
  uint32_t magic;
  uint32_t abi;
  uint64_t cfg_hash;
  int32_t batch;
  int32_t n_layers;
  uint64_t stream_stride;
};
static_assert(sizeof(StateHeader) <= kHeaderBytes, "header too large");

// Byte offsets inside one (layer, sequence) stream block.
struct StreamOffsets {
  long long pos, win_k, win_v, far, field, ring_sum, ring;
  long long stride;
};

struct DecodeParams {
  const void* q;
  const void* k;
  const void* v;
  float* out;
  unsigned char* state;
  const float* slots;       // [L][64][H]
  const float* slot_norm;   // [L][64], clamped at kNormFloor
  const float* alpha_layer; // [L]
  const unsigned char* slot_img;  // pre-split bf16 slot blocks (batch-tiled decode)
  int* err;
  uint64_t cfg_hash;
  StreamOffsets so;
  int L, B, nq, nkv, K, H, G, CS, HPC;
  int l0, Lc;            // layers l0 .. l0+Lc-1 of the state are served
  const int* seq_ids;    // [n_seq] sequences served (device), or null: 0 .. n_seq-1
  int n_seq;
  int NGm;          // most KV heads any CTA needs
  int smem_budget;  // shared-memory bytes the plan may use (window staged if it fits)
  int tile_smem;    // dynamic shared memory of the batch-tiled decode
  float gamma_far, alpha_far, ema_gamma, inv_temp, clip_eps, score_scale;
};

constexpr int kDecodeSmemBudget = 112 * 1024;  // keeps two decode CTAs per SM

// Shared-memory plan of the prefill kernel (byte offsets).
struct PrefillPlan {
  int bars, xs, halo, fcar, sst, sagg, sega, ml;  // persistent regions
  int u0;                                   // start of the union below
  int tc;                                   // near field on the tensor cores (bf16, k <= 16)
  int qst, kb, vb;                          // near-field staging (phase 1, CUDA-core near field)
  int qa, kvp, pa;                          // near-field MMA operands (phase 1, tensor-core near field)
  int sl, part, wts, semc;                  // pool buffers (phase 2)
  int KB;                                   // rows per staged key/value block
  int total;
};

struct PrefillParams {
  const void* q;
  const void* k;
  const void* v;
  float* out;
  unsigned char* state;
  unsigned char* ws;
  const float* slots;
  const float* slot_norm;
  const float* alpha_layer;
  const unsigned char* slot_img;  // pre-split bf16 slot blocks
  int* err;
  uint64_t cfg_hash;
  StreamOffsets so;
  long long n;              // tokens per stream in this call
  int L, B, nq, nkv, K, H, G, CS, HPC;
  int l0;                   // first layer of the state served (streams are l0*B + ...)
  int NGm;                  // most KV heads any CTA needs
  int KB;                   // rows per staged key/value block
  int tiles_per_stream, n_streams;
  long long n_tiles;
  // workspace byte offsets
  long long ws_fs_agg, ws_fs_incl, ws_ff_agg, ws_ff_incl;
  long long ws_agg_s, ws_incl_s, ws_agg_f, ws_incl_f, ws_halo;
  float gamma_far, alpha_far, ema_gamma, inv_temp, clip_eps, score_scale;
  unsigned spin_limit;
  long long withhold_tile;
  PrefillPlan plan;
};

// Workspace layout for a prefill call (bytes).
struct PrefillWorkspace {
  long long fs_agg, fs_incl, ff_agg, ff_incl, flags_end;  // [0, flags_end) cleared per call
  long long agg_s, incl_s, agg_f, incl_f, halo, total;
};

inline long long align256(long long x) { return (x + 255) & ~255LL; }

// Launchers (return the CUDA error of the launch).
cudaError_t launch_decode(const DecodeParams& p, int in_dtype, int head_dim, cudaStream_t s);
cudaError_t launch_decode_tile(const DecodeParams& p, int in_dtype, int head_dim, cudaStream_t s);
cudaError_t decode_tile_prepare(int device);
size_t decode_tile_smem_bytes(int HPC, int head_dim, size_t limit);
int decode_tile_max_active_clusters(int cs, size_t smem, int in_dtype, int head_dim);
cudaError_t launch_prefill(const PrefillParams& p, int in_dtype, int head_dim, cudaStream_t s);
bool plan_prefill(int HPC, int D, int esz, int NGm, int K, size_t budget, bool tc, PrefillPlan* out);
cudaError_t prefill_prepare(int device);
cudaError_t decode_prepare(int device);
size_t decode_smem_bytes(int HPC, int head_dim, int esz, int NGm, int K, int budget);
int prefill_max_active_clusters(int cs, size_t smem, int in_dtype, int head_dim);
int decode_max_active_clusters(int cs, size_t smem, int in_dtype, int head_dim);
size_t prefill_smem_limit(int device);
cudaError_t launch_write_header(unsigned char* state, StateHeader h, cudaStream_t s);
cudaError_t launch_slot_norms(const float* slots, float* norms, int L, int H, cudaStream_t s);
// Pre-split bf16 slot blocks for the prefill pool MMAs ([L][H/64][hi, lo]
// 64 x 64 blocks, 8 KB each); H must be a multiple of 64.
cudaError_t launch_slot_image(const float* slots, unsigned char* img, int L, int H, cudaStream_t s);

}  // namespace sfa
