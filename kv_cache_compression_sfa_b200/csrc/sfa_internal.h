// sfa_internal.h — layouts and kernel parameter blocks shared by the host
// launch layer (sfa_api.cu) and the kernels (sfa_decode.cu, sfa_prefill.cu).
//
// Sources (web pages):
//   [P1] "Signal Field Attention (SFA)：8KB代码实现4.16倍推理加速与248倍内存压缩"
//   [P2] "Signal Field Attention (SFA)" (project README page)
//   [P3] "Dalin Soma SFA基于信号场注意力机制的神经网络推理加速框架"
#pragma once

#include <cuda.h>
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
constexpr int kHalo = kRing - 1;          // x rows a token needs from before its tile
constexpr int kPrefillThreads = 256;
constexpr int kDecodeThreads = 256;
constexpr long long kFusedMinTilesPerSm = 4;  // prefill calls from this many tiles per SM take the fused kernel
constexpr int kDecodeTileMinSeqs = 64;      // batch-tiled decode from this many sequences per call
constexpr int kDecodeTileHeads = 8;         // most query heads per KV head it serves
constexpr int kDecodeTileChunk = 16;        // window slots per staged chunk

constexpr unsigned kDefaultSpinLimit = 1u << 21;  // polls of a bounded wait

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

// Plans of the batch-tiled decode (byte offsets and sizes; see
// sfa_decode_tile.cu): its near-field kernel and its pool kernel.
struct TilePlan {
  int kcb;          // window slots per staged chunk
  int hq, hkt, hvt, hs, hdr_bytes;  // per-warp header: q of the KV head's query heads, K_t, V_t, S
  int chunk_bytes;  // a staged window chunk: keys, then values
  int warp_bytes;   // per warp: two headers and two chunks
  int near_warps;   // warps of a near-field CTA
  int near_rows;    // sequences of a near-field CTA
  int near_smem;    // its dynamic shared memory
  int pool_smem;    // dynamic shared memory of the pool kernel
};

struct DecodeParams {
  const void* q;
  const void* k;
  const void* v;
  float* out;               // fp32 result (SFA_OUT_F32), where the batch-tiled decode keeps x
  void* res;                // result in the output mode's dtype
  int out_mode;             // sfa_out_mode
  unsigned char* state;
  const float* slots;       // [L][64][H]
  const float* slot_norm;   // [L][64], clamped at kNormFloor
  const float* alpha_layer; // [L]
  const unsigned char* slot_img;  // pre-split bf16 slot blocks (batch-tiled decode)
  const float* slot_dec;          // [L][CS][64][HS + 4] slot slice of every decode CTA
  int* err;
  uint64_t cfg_hash;
  StreamOffsets so;
  int L, B, nq, nkv, K, H, G, CS, HPC;
  int l0, Lc;            // layers l0 .. l0+Lc-1 of the state are served
  const int* seq_ids;    // [n_seq] sequences served (device), or null: 0 .. n_seq-1
  int n_seq;
  int NGm;          // most KV heads any CTA needs
  int smem_budget;  // shared-memory bytes the plan may use (window staged if it fits)
  TilePlan tp;      // shared-memory plan of the batch-tiled decode
  int inputs_early; // q, K_t, V_t may be fetched before the wait for the previous kernel
  float gamma_far, alpha_far, ema_gamma, inv_temp, clip_eps, score_scale;
};

constexpr int kDecodeSmemBudget = 112 * 1024;  // keeps two decode CTAs per SM

// Shared-memory plan of the prefill near-field kernel (byte offsets).  Each
// stage holds one tile's queries of one head and the keys and values of its
// span (positions t0-k .. t0+T-1), rows padded by 16 bytes.
struct NearPlan {
  int tc;                 // near field on the tensor cores (bf16 inputs, k <= 16)
  int fused;              // tensor cores: near field and pool scores in one kernel (fused_kernel)
  int stages;             // 2 or 1 staged buffers; 0: keys and values read from global memory
  int row;                // CUDA cores: padded bytes of one staged row
  int q[2], k[2], v[2];   // stage offsets (tensor cores: MMA operand blocks)
  int pa;                 // tensor cores: P blocks (hi, lo)
  int ga;                 // tensor cores: far-field weight blocks G (hi, lo)
  int xs;                 // CUDA cores: x tile [kTile][D + 4] fp32
  int total;
};

struct PrefillParams {
  const void* q;
  const void* k;
  const void* v;
  float* out;               // x between the kernels: the result buffer (SFA_OUT_F32) or workspace
  void* res;                // result in the output mode's dtype
  int out_mode;             // sfa_out_mode
  unsigned char* state;
  unsigned char* ws;
  const float* slots;
  const float* slot_norm;
  const float* alpha_layer;
  const unsigned char* slot_img;  // pre-split bf16 slot blocks
  int* err;
  uint64_t cfg_hash;
  StreamOffsets so;
  long long n;              // tokens per stream in this call (row pitch of q, k, v, out)
  const int* lens;          // [B] tokens of each sequence (ragged call, device), or null: all n
  int L, B, nq, nkv, K, H, G;
  int l0;                   // first layer of the state served (streams are l0*B + ...)
  int tiles_per_stream, n_streams;
  int n_seg, tps;           // near field (or fused kernel): segments per stream, tiles per segment
  int nseg_out, tps_out;    // output kernel: segments per stream, tiles per segment
  // workspace byte offsets: stream positions, S at the end of the call, pool
  // weights, far-field state at every tile start, x (output modes other
  // than SFA_OUT_F32)
  long long ws_pos, ws_sfin, ws_w, ws_sst, ws_x;
  long long ws_fagg, ws_halo;  // EMA field over each tile from zero; x rows before each output segment
  float gamma_far, alpha_far, ema_gamma, inv_temp, clip_eps, score_scale;
  unsigned spin_limit;      // polls of a bounded wait before it gives up
  long long withhold_tile;  // test hook: this tile's pool CTA waits on a barrier nothing completes
  NearPlan near;
  int pool_smem, out_smem;
};

// Tensor maps of one prefill call's q, k and v for the tensor-core near field:
// 3-D views (head dim, head, token row over all streams of the call) whose
// 8-element x 1 x T-row boxes land as one column of core matrices.
struct NearMaps {
  CUtensorMap q, k, v;
};

// Workspace layout for a prefill call (bytes); nothing in it needs clearing.
struct PrefillWorkspace {
  long long pos;    // [streams] int64 position at the start of the call
  long long sfin;   // [streams][n_kv][d] fp32 far state at the end of the call
  long long w;      // [streams * tiles][hi, lo] 64 x 64 bf16 pool-weight blocks
  long long sst;    // [streams][tiles][n_kv][d] fp32 far state at every tile start
  long long x;      // [streams][n][H] fp32 x when the result is not fp32 x + enhancement (else 0)
  long long fagg;   // [streams][tiles][H] fp32 EMA field over each tile, from zero
  long long halo;   // [streams][output segments][15][H] fp32 x rows before each output segment
  long long total;
};

inline long long align256(long long x) { return (x + 255) & ~255LL; }

// Launchers (return the CUDA error of the launch).
cudaError_t launch_decode(const DecodeParams& p, int in_dtype, int head_dim, cudaStream_t s);
cudaError_t launch_decode_tile(const DecodeParams& p, int in_dtype, int head_dim, cudaStream_t s);
cudaError_t decode_tile_prepare(int device);
// Plan of the batch-tiled decode within `limit` bytes of shared memory;
// false if none fits or the configuration is outside it (more than
// kDecodeTileHeads query heads per KV head, hidden not a multiple of 64).
bool plan_decode_tile(int H, int head_dim, int esz, int G, int K, size_t limit, TilePlan* out);
cudaError_t launch_prefill(const PrefillParams& p, int in_dtype, int head_dim, cudaStream_t s);
// Near-field plan for head_dim D, input element size esz and window K within
// `limit` bytes of shared memory, on the tensor cores if tc (bf16, K <= 16),
// there fused with the pool scores if fused; false if none fits.
bool plan_near(int D, int esz, int K, size_t limit, bool tc, bool fused, NearPlan* out);
int prefill_pool_smem();
int prefill_out_smem();
cudaError_t prefill_prepare(int device);
cudaError_t decode_prepare(int device);
size_t decode_smem_bytes(int HPC, int head_dim, int esz, int NGm, int nkv, int K, int budget);
int decode_max_active_clusters(int cs, size_t smem, int in_dtype, int head_dim);
size_t prefill_smem_limit(int device);
cudaError_t launch_write_header(unsigned char* state, StateHeader h, cudaStream_t s);
cudaError_t launch_slot_norms(const float* slots, float* norms, int L, int H, cudaStream_t s);
// Pre-split bf16 slot blocks for the prefill pool MMAs ([L][H/64][hi, lo]
// 64 x 64 blocks, 8 KB each); H must be a multiple of 64.
cudaError_t launch_slot_image(const float* slots, unsigned char* img, int L, int H, cudaStream_t s);

}  // namespace sfa
