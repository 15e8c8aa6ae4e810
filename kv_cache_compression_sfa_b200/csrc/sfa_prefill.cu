// sfa_prefill.cu — SFA prefill: n tokens per (layer, sequence) stream,
// each kernel parallel over independent work units with no waits between
// CTAs, chained by programmatic dependent launch.
//
// Sources (web pages):
//   [P1] "Signal Field Attention (SFA)：8KB代码实现4.16倍推理加速与248倍内存压缩"
//        §2.1 eqs. O_near, S_t, O; §2.2 O(k·d) window state.
//   [P3] "Dalin Soma SFA基于信号场注意力机制的神经网络推理加速框架"
//        §2.1 channels 1–3, §2.2 fusion, clip and alpha_layer, §2.4 ring mean.
//
// 0. far_agg_kernel / far_carry_kernel: the far-field EWMA S [P1 §2.1 eq.
//    S_t] at every tile start of kTile tokens, as a two-level scan: one
//    aggregate of the evicted keys per tile (independent terms), then one
//    fold in tile order per (stream, KV head, dim).
// 1. The near field [P1 §2.1 eq. O_near] and x = O_near + alpha_far * S
//    [P1 §2.1 eq. O], then the pool scores, softmax(cos/T) weights and the
//    EMA field over each tile [P3 §2.1 channels 2-3], by one of:
//    * fused_kernel (bf16, k <= 16, large calls): one CTA per (stream,
//      segment of tiles) walks every head of each tile; queries and the
//      key/value span arrive by tensor copies, the band scores, P.V + G.K,
//      the pool scores and the field aggregates are tcgen05 MMAs with
//      accumulators in tensor memory, and warp-specialized roles hand off
//      through mbarriers.  x is written once, for step 2.
//    * near_tc_kernel (bf16, k <= 16) or near_kernel (CUDA cores), one CTA
//      per (stream, query head, segment of tiles), writing x; then
//      pool_kernel, one CTA per (stream, tile), reads x back for the
//      scores (tcgen05, split bf16 operands), weights and field aggregates.
//    The weights go to the workspace as split bf16 blocks in the MMA operand
//    layout; x lives in `out` (fp32 results) or in the workspace.
// 2. out_kernel, one CTA per (stream, 64 hidden columns, segment of tiles),
//    walks its tiles in order: sem[T x 64] = w . slot_chunk on the tensor
//    cores; per column the ring sum over the last 16 x (a sliding sum, the
//    15 rows before the tile kept from the previous one or, at a segment
//    start, from the halo rows step 1 kept) and the EMA field (from the fold
//    of the earlier tiles' aggregates), four token segments per column
//    joined by their carries; the fusion, clip and scale [P3 §2.1, §2.2]
//    give the result in the output mode's form.  At the stream's end: ring
//    slots, ring sum, field; one CTA per stream also writes the window, S
//    and the position.
//
// Each kernel waits for its predecessor before touching what that one
// writes.  Every wait on a copy, MMA or role hand-off is bounded; a wait
// that runs out latches SFA_ERR_DEVICE_TIMEOUT and the kernel still
// finishes.
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstring>

#include "sfa_common.cuh"
#include "sfa_umma.cuh"

namespace sfa {
namespace {

constexpr int NT = kPrefillThreads;
constexpr int NW = NT / 32;
constexpr int kTmemCols = 64;          // one 64 x 64 fp32 accumulator
constexpr int kSeg = 4;                // token segments per column in out_kernel
constexpr int kSegLen = kTile / kSeg;
constexpr int kScStride = kSlots + 1;  // padded row of the staged scores
constexpr int kXsPad = 4;              // x tile row padding (floats) in near_kernel
static_assert(kTile == kBlk, "tile tokens are the M of the pool MMAs");
static_assert(kSegLen >= kRing, "a segment's ring window reaches back at most one segment");

// Every kernel checks the state header (same answer in every CTA).
__device__ __forceinline__ bool header_matches(const PrefillParams& p) {
  const uint4 h0v = __ldcg(reinterpret_cast<const uint4*>(p.state));
  const uint4 h1v = __ldcg(reinterpret_cast<const uint4*>(p.state + 16));
  StateHeader hd;
  reinterpret_cast<uint4*>(&hd)[0] = h0v;
  reinterpret_cast<uint4*>(&hd)[1] = h1v;
  return hd.magic == kMagic && hd.cfg_hash == p.cfg_hash && hd.batch == p.B && hd.n_layers == p.L;
}

__device__ __forceinline__ unsigned char* stream_block(const PrefillParams& p, int s) {
  return p.state + kHeaderBytes + (static_cast<long long>(p.l0) * p.B + s) * p.so.stride;
}

// Tokens that call-relative stream s folds in: the call's n, or for a
// ragged call its sequence's own count (a count outside 0 .. n counts as 0;
// far_agg_kernel latches it).  Inputs and outputs keep a row pitch of n.
__device__ __forceinline__ long long stream_len(const PrefillParams& p, int s) {
  if (!p.lens) return p.n;
  const int v = __ldg(p.lens + (s % p.B));
  return (v < 0 || v > p.n) ? 0 : v;
}

// ======================================================================
// 0. far-field state at every tile start [P1 §2.1 eq. S_t]
// ======================================================================
// S folds one evicted key per token once the position reaches k, so over a
// tile of Tt tokens S_end = gamma^ev S_start + agg with
//   agg = sum over evicting tokens r of (1-gamma) gamma^(Tt-1-r) K_{t0+r-k},
// ev the number of evicting tokens.  far_agg_kernel forms agg for every
// tile in parallel (independent terms); far_carry_kernel folds them in tile
// order per (stream, KV head, dim) and stores S at every tile start (in
// place of agg) and at the end of the call.

template <typename Tin, int D>
__global__ void __launch_bounds__(NT) far_agg_kernel(const PrefillParams p) {
  constexpr int VE = Load16<Tin>::N;  // dims per 16-byte load
  constexpr int kQ = 4;               // token quarters of a tile
  constexpr int kQLen = kTile / kQ;
  const int tile = blockIdx.x, s = blockIdx.y, tid = threadIdx.x;
  __shared__ int s_ok;
  __shared__ long long s_pos;
  __shared__ float s_w[kTile];
  extern __shared__ __align__(16) unsigned char smb[];  // [kQ][n_kv * D] quarter sums

  pdl_trigger();
  pdl_wait();  // the state may be written by the previous kernel of the stream
  unsigned char* blk = stream_block(p, s);
  if (tid == 0) {
    s_ok = header_matches(p);
    s_pos = __ldcg(reinterpret_cast<const long long*>(blk + p.so.pos));
  }
  __syncthreads();
  if (!s_ok) {  // uniform over the grid; every later kernel of the call sees it too
    if (tid == 0 && tile == 0 && s == 0) latch_error(p.err, SFA_ERR_STATE_MISMATCH);
    return;
  }
  const long long pos0 = s_pos;
  const long long ns = stream_len(p, s);
  if (tid == 0 && tile == 0) {
    reinterpret_cast<long long*>(p.ws + p.ws_pos)[s] = pos0;
    if (p.lens) {
      const int v = __ldg(p.lens + (s % p.B));
      if (v < 0 || v > p.n) latch_error(p.err, SFA_ERR_INVALID_ARG);
    }
  }
  const int K = p.K, nkv = p.nkv;
  const long long t0 = pos0 + static_cast<long long>(tile) * kTile;
  // tokens of this tile (<= 0 past a ragged stream's end: nothing evicts)
  const int Tt = static_cast<int>(min(static_cast<long long>(kTile), ns - static_cast<long long>(tile) * kTile));
  if (tid < kTile)
    s_w[tid] = (tid < Tt && t0 + tid >= K) ? (1.0f - p.gamma_far) * powf(p.gamma_far, static_cast<float>(Tt - 1 - tid)) : 0.f;
  __syncthreads();
  const Tin* win_k = reinterpret_cast<const Tin*>(blk + p.so.win_k);
  const Tin* kin = static_cast<const Tin*>(p.k) + static_cast<long long>(s) * p.n * nkv * D;
  const int ne = nkv * D, nv = ne / VE;
  float* part = reinterpret_cast<float*>(smb);
  // Work item (16-byte dim group v, token quarter q): the quarter's 16 keys
  // all in flight at once.
  for (int it = tid; it < nv * kQ; it += NT) {
    const int v = it % nv, q = it / nv;
    const int g = (v * VE) / D, d0 = (v * VE) % D;
    uint4 raw[kQLen];  // raw 16-byte loads, all in flight; unpacked at the multiply-add
#pragma unroll
    for (int u = 0; u < kQLen; ++u) {
      const int r = q * kQLen + u;
      const long long t = t0 + r;
      // evicted position; tokens that evict nothing read their own key (weight 0)
      const long long j = (r < Tt && t >= K) ? t - K : t0;
      const Tin* row = j >= pos0 ? kin + ((j - pos0) * nkv + g) * D : win_k + ((j % K) * nkv + g) * D;
      raw[u] = *reinterpret_cast<const uint4*>(row + d0);
    }
    float acc[VE];
#pragma unroll
    for (int e = 0; e < VE; ++e) acc[e] = 0.f;
#pragma unroll
    for (int u = 0; u < kQLen; ++u) {
      const float w = s_w[q * kQLen + u];
      float kv[VE];
      Load16<Tin>::run(reinterpret_cast<const Tin*>(&raw[u]), kv);
#pragma unroll
      for (int e = 0; e < VE; ++e) acc[e] = fmaf(w, kv[e], acc[e]);
    }
#pragma unroll
    for (int e = 0; e < VE; ++e) part[q * ne + v * VE + e] = acc[e];
  }
  __syncthreads();
  float* agg = reinterpret_cast<float*>(p.ws + p.ws_sst) +
               (static_cast<long long>(s) * p.tiles_per_stream + tile) * ne;
  for (int e = tid; e < ne; e += NT)  // quarters added in order
    agg[e] = ((part[e] + part[ne + e]) + part[2 * ne + e]) + part[3 * ne + e];
}

__global__ void __launch_bounds__(NT) far_carry_kernel(const PrefillParams p) {
  const int s = blockIdx.y;
  const int e = blockIdx.x * NT + threadIdx.x;
  __shared__ int s_ok;
  pdl_trigger();
  pdl_wait();  // tile aggregates from far_agg_kernel
  if (threadIdx.x == 0) s_ok = header_matches(p);
  __syncthreads();
  const int ne = p.nkv * (p.H / p.nq);
  if (!s_ok || e >= ne) return;
  const long long pos0 = reinterpret_cast<const long long*>(p.ws + p.ws_pos)[s];
  const long long ns = stream_len(p, s);
  const float* far = reinterpret_cast<const float*>(stream_block(p, s) + p.so.far);
  float S = far[e];
  float* a = reinterpret_cast<float*>(p.ws + p.ws_sst) + static_cast<long long>(s) * p.tiles_per_stream * ne + e;
  const float gf = p.gamma_far, g64 = powf(gf, static_cast<float>(kTile));
  const int tiles = p.tiles_per_stream, K = p.K;
  constexpr int kChunk = 8;  // aggregates in flight per thread
  for (int t8 = 0; t8 < tiles; t8 += kChunk) {
    float av[kChunk];
#pragma unroll
    for (int u = 0; u < kChunk; ++u) av[u] = (t8 + u < tiles) ? a[static_cast<long long>(t8 + u) * ne] : 0.f;
#pragma unroll
    for (int u = 0; u < kChunk; ++u) {
      const int i = t8 + u;
      if (i < tiles) {
        const long long t0 = pos0 + static_cast<long long>(i) * kTile;
        const long long Tt = min(static_cast<long long>(kTile), ns - static_cast<long long>(i) * kTile);
        const long long ev = max(0LL, t0 + Tt - max(t0, static_cast<long long>(K)));
        const float gev = ev == kTile ? g64 : powf(gf, static_cast<float>(ev));
        a[static_cast<long long>(i) * ne] = S;
        S = fmaf(gev, S, av[u]);
      }
    }
  }
  reinterpret_cast<float*>(p.ws + p.ws_sfin)[static_cast<long long>(s) * ne + e] = S;
}

// ======================================================================
// 1. near field, far field and x
// ======================================================================

// Near field of the tile's tokens for one query head [P1 §2.1 eq. O_near]:
// LP lanes serve a token; lane a scores key base+a in full, online softmax
// across chunks of LP keys, then P·V with the LP lanes over head dims; the
// result is added to the token's row of the x tile (which holds alpha*S).
// krow(j)/vrow(j): key/value row of absolute position j.
template <typename Tin, int D, int LP, typename KR, typename VR>
__device__ __forceinline__ void near_tile(const unsigned char* qs, int RB, float* xs, int Tt,
                                          long long t0, int K, float scale, int warp, int lane,
                                          KR krow, VR vrow) {
  constexpr int PPW = 32 / LP;  // tokens per warp
  constexpr int EPL = D / LP;   // head dims per lane in P·V
  constexpr int VE = Load16<Tin>::N;
  constexpr int XS = D + kXsPad;
  const int sub = lane / LP, sl = lane % LP;
  const int gbase = sub * LP;
  for (int rb = warp * PPW; rb < Tt; rb += NW * PPW) {
    const int r = rb + sub;
    const bool live = r < Tt;
    const long long pt = t0 + r;
    const long long lo = pt - K + 1 > 0 ? pt - K + 1 : 0;
    const int cnt = live ? static_cast<int>(pt - lo + 1) : 0;
    int cnt_max = cnt;  // the tokens of a warp run the same number of chunks
    if (LP < 32) cnt_max = max(cnt_max, __shfl_xor_sync(0xffffffffu, cnt_max, 16));
    const Tin* qrow = reinterpret_cast<const Tin*>(qs + (live ? r : 0) * RB);
    float m = -INFINITY, den = 0.f, o[EPL];
#pragma unroll
    for (int e = 0; e < EPL; ++e) o[e] = 0.f;
    for (int base = 0; base < cnt_max; base += LP) {
      const int cc = max(0, min(LP, cnt - base));  // this token's keys in the chunk
      float sc = -INFINITY;
      if (sl < cc) {
        const Tin* kr = krow(lo + base + sl);
        float acc[4] = {0.f, 0.f, 0.f, 0.f};  // independent chains
#pragma unroll
        for (int i = 0; i < D; i += VE) {
          float kv[VE], qv[VE];
          Load16<Tin>::run(kr + i, kv);
          Load16<Tin>::run(qrow + i, qv);
#pragma unroll
          for (int e = 0; e < VE; ++e) acc[e & 3] = fmaf(qv[e], kv[e], acc[e & 3]);
        }
        sc = ((acc[0] + acc[1]) + (acc[2] + acc[3])) * scale;
      }
      float cm = sc;
#pragma unroll
      for (int off = LP / 2; off > 0; off >>= 1) cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, off));
      const float mn = (cc > 0) ? fmaxf(m, cm) : m;
      const float corr = (cc > 0) ? expf(m - mn) : 1.f;
      const float pj = (sl < cc) ? expf(sc - mn) : 0.f;
      float ps = pj;
#pragma unroll
      for (int off = LP / 2; off > 0; off >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
      den = fmaf(den, corr, ps);
#pragma unroll
      for (int e = 0; e < EPL; ++e) o[e] *= corr;
      const int cmax = min(LP, cnt_max - base);
      for (int c = 0; c < cmax; ++c) {
        const float pc = __shfl_sync(0xffffffffu, pj, gbase + c);
        if (c < cc) {
          float vv[EPL];
          VecLoad<Tin, EPL>::run(vrow(lo + base + c) + sl * EPL, vv);
#pragma unroll
          for (int e = 0; e < EPL; ++e) o[e] = fmaf(pc, vv[e], o[e]);
        }
      }
      m = mn;
    }
    if (live) {
      const float inv = 1.f / den;
      float* xr = xs + r * XS + sl * EPL;
#pragma unroll
      for (int e = 0; e < EPL; ++e) xr[e] = fmaf(o[e], inv, xr[e]);
    }
  }
}

template <typename Tin, int D>
__global__ void __launch_bounds__(NT, 2) near_kernel(const PrefillParams p) {
  constexpr int ESZ = static_cast<int>(sizeof(Tin));
  constexpr int C16 = D * ESZ / 16;  // 16-byte chunks of one head row
  constexpr int XS = D + kXsPad;
  const int h = blockIdx.x % p.nq, seg = blockIdx.x / p.nq;  // query head, segment of tiles
  const int s = blockIdx.y;                                   // call-relative stream
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  extern __shared__ __align__(16) unsigned char smb[];
  const NearPlan& np = p.near;
  __shared__ int s_ok;
  __shared__ long long s_pos;

  pdl_trigger();
  pdl_wait();  // far state at the tile starts from far_carry_kernel
  unsigned char* blk = stream_block(p, s);
  if (tid == 0) {
    s_ok = header_matches(p);
    s_pos = reinterpret_cast<const long long*>(p.ws + p.ws_pos)[s];
  }
  __syncthreads();
  if (!s_ok) return;  // latched by far_agg_kernel
  const long long pos0 = s_pos;
  const long long ns = stream_len(p, s);  // tokens of this stream in the call
  const int K = p.K, nkv = p.nkv, g = h / p.G;
  const Tin* win_k = reinterpret_cast<const Tin*>(blk + p.so.win_k);
  const Tin* win_v = reinterpret_cast<const Tin*>(blk + p.so.win_v);
  const float* sst = reinterpret_cast<const float*>(p.ws + p.ws_sst) +
                     static_cast<long long>(s) * p.tiles_per_stream * nkv * D + g * D;
  const long long in_row0 = static_cast<long long>(s) * p.n;  // first input row of the stream
  const Tin* qin = static_cast<const Tin*>(p.q) + in_row0 * p.nq * D;
  const Tin* kin = static_cast<const Tin*>(p.k) + in_row0 * nkv * D;
  const Tin* vin = static_cast<const Tin*>(p.v) + in_row0 * nkv * D;
  // Key/value row of absolute position j >= 0 for KV head g: from the input
  // if it belongs to this call, else from window slot j mod k (the state
  // holds positions pos0-k .. pos0-1).
  auto krow_g = [&](long long j) -> const Tin* {
    return j >= pos0 ? kin + ((j - pos0) * nkv + g) * D : win_k + ((j % K) * nkv + g) * D;
  };
  auto vrow_g = [&](long long j) -> const Tin* {
    return j >= pos0 ? vin + ((j - pos0) * nkv + g) * D : win_v + ((j % K) * nkv + g) * D;
  };
  const int RB = np.row;
  float* xs = reinterpret_cast<float*>(smb + np.xs);

  // Copies of tile i into stage st: its queries and (staged plans) the key
  // and value rows of positions t0-k .. t0+Tt-1; positions before 0 are
  // never read and stay unloaded.
  auto issue = [&](int i, int st) {
    const long long t0 = pos0 + static_cast<long long>(i) * kTile;
    const int Tt = static_cast<int>(min(static_cast<long long>(kTile), ns - static_cast<long long>(i) * kTile));
    unsigned char* qs = smb + np.q[st];
    for (int c = tid; c < Tt * C16; c += NT) {
      const int r = c / C16, u = c % C16;
      cp_async16(qs + r * RB + u * 16,
                 reinterpret_cast<const unsigned char*>(qin + ((t0 - pos0 + r) * p.nq + h) * D) + u * 16);
    }
    if (np.stages > 0) {
      unsigned char* ks = smb + np.k[st];
      unsigned char* vs = smb + np.v[st];
      const int R = Tt + K;
      for (int c = tid; c < R * C16; c += NT) {
        const int r = c / C16, u = c % C16;
        const long long j = t0 - K + r;
        if (j < 0) continue;
        cp_async16(ks + r * RB + u * 16, reinterpret_cast<const unsigned char*>(krow_g(j)) + u * 16);
        cp_async16(vs + r * RB + u * 16, reinterpret_cast<const unsigned char*>(vrow_g(j)) + u * 16);
      }
    }
    cp_async_commit();
  };

  const float gf = p.gamma_far, af = p.alpha_far;
  // this CTA's tiles (a ragged stream may end before them)
  const int tiles_s = static_cast<int>((ns + kTile - 1) / kTile);
  const int i0 = seg * p.tps, tiles = min(min(p.tiles_per_stream, tiles_s), i0 + p.tps);
  if (i0 < tiles) issue(i0, 0);
  for (int i = i0; i < tiles; ++i) {
    const int st = (np.stages == 2) ? ((i - i0) & 1) : 0;
    // S of KV head g, dim tid, at the tile start
    float sreg = (tid < D) ? sst[static_cast<long long>(i) * nkv * D + tid] : 0.f;
    if (np.stages == 2 && i + 1 < tiles) {
      issue(i + 1, st ^ 1);  // that stage was released at the end of tile i-1
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const long long t0 = pos0 + static_cast<long long>(i) * kTile;
    const int Tt = static_cast<int>(min(static_cast<long long>(kTile), ns - static_cast<long long>(i) * kTile));
    const unsigned char* qs = smb + np.q[st];
    const unsigned char* ks = smb + np.k[st];
    const unsigned char* vs = smb + np.v[st];
    const bool staged = np.stages > 0;

    // Far field [P1 §2.1 eq. S_t]: token t0+r evicts position t0+r-k (span
    // row r) once t0+r >= k; x starts as alpha_far * S_t.
    if (tid < D) {
      const int r_ev = static_cast<int>(max(0LL, min(static_cast<long long>(Tt), K - t0)));
      for (int r = 0; r < r_ev; ++r) xs[r * XS + tid] = af * sreg;
      if (staged) {
        const Tin* col = reinterpret_cast<const Tin*>(ks) + tid;
        const int pitch = RB / ESZ;
        for (int r = r_ev; r < Tt; ++r) {
          sreg = ewma(gf, sreg, to_f32<Tin>(col[r * pitch]));
          xs[r * XS + tid] = af * sreg;
        }
      } else {
        for (int r = r_ev; r < Tt; ++r) {
          sreg = ewma(gf, sreg, to_f32<Tin>(krow_g(t0 + r - K)[tid]));
          xs[r * XS + tid] = af * sreg;
        }
      }
    }
    __syncthreads();

    // Near field, added onto alpha_far * S.
    const long long span0 = t0 - K;  // position of span row 0
    auto krow_s = [&](long long j) -> const Tin* {
      return reinterpret_cast<const Tin*>(ks + static_cast<int>(j - span0) * RB);
    };
    auto vrow_s = [&](long long j) -> const Tin* {
      return reinterpret_cast<const Tin*>(vs + static_cast<int>(j - span0) * RB);
    };
    if (staged) {
      if (K <= 16) near_tile<Tin, D, 16>(qs, RB, xs, Tt, t0, K, p.score_scale, warp, lane, krow_s, vrow_s);
      else near_tile<Tin, D, 32>(qs, RB, xs, Tt, t0, K, p.score_scale, warp, lane, krow_s, vrow_s);
    } else {
      if (K <= 16) near_tile<Tin, D, 16>(qs, RB, xs, Tt, t0, K, p.score_scale, warp, lane, krow_g, vrow_g);
      else near_tile<Tin, D, 32>(qs, RB, xs, Tt, t0, K, p.score_scale, warp, lane, krow_g, vrow_g);
    }
    __syncthreads();

    // x rows into out (this head's columns).
    float* orow0 = p.out + (in_row0 + (t0 - pos0)) * p.H + h * D;
    for (int c = tid; c < Tt * (D / 4); c += NT) {
      const int r = c / (D / 4), c4 = (c % (D / 4)) * 4;
      *reinterpret_cast<float4*>(orow0 + static_cast<long long>(r) * p.H + c4) =
          *reinterpret_cast<const float4*>(xs + r * XS + c4);
    }
    __syncthreads();  // the stage and the x tile are free again
    if (np.stages != 2 && i + 1 < tiles) issue(i + 1, 0);
  }
}

// Near field and far field on the tensor cores (bf16 inputs, k <= 16).
// Per tile, with the span fixed at positions t0-16 .. t0+63 (kNS rows):
//   scores[64 x kNS] = Q . K_span^T (tensor memory, columns 0 .. kNS-1;
//   bf16 products are exact, fp32 accumulation) [P1 §2.1 eq. O_near];
//   softmax over the band of each row (token r sees span rows r+17-k ..
//   r+16, none before position 0), P split into bf16 hi + lo;
//   X[64 x D] = P . V_span + G . K_span (columns kTmemO ..), each product
//   as hi + lo of the split left operand.
// The far field [P1 §2.1 eq. S_t] inside a tile is linear in the keys it
// evicts: with r_ev the first token of the tile that evicts (token r evicts
// position t0+r-k, span row r+16-k) and S0 the state at the tile start,
//   S_r = gamma^m(r) S0 + sum_{r_ev <= j <= r} (1-gamma) gamma^(r-j) e_j,
// m(r) = max(0, r - r_ev + 1).  G[r][c] = alpha_far (1-gamma) gamma^(r-j)
// for span row c = j+16-k holds the second term, so X = O_near + alpha_far
// (S_r - gamma^m(r) S0) and the epilogue adds alpha_far gamma^m(r) S0
// [P1 §2.1 eq. O]; S0 comes from far_carry_kernel.
// Operand blocks use the core-matrix layout of sfa_umma.cuh; in the key and
// value blocks the 8-dim groups are kDStr bytes apart, each a column of
// kNS core-matrix rows that one tensor copy fills.  The key and value
// blocks are the MN-major B of G.K and P.V.  Tensor copies need 128-byte
// aligned shared-memory destinations: the blocks start at multiples of 128.
constexpr int kNS = kTile + 16;
constexpr int kDStr = (kNS / 8) * 128;
constexpr int kTmemNear = 256;
constexpr int kTmemO = 128;

__device__ __forceinline__ int kv_off(int c, int d) {
  return (d >> 3) * kDStr + (c >> 3) * 128 + (c & 7) * 16 + (d & 7) * 2;
}

template <int D>
__global__ void __launch_bounds__(NT, 2)
near_tc_kernel(const __grid_constant__ PrefillParams p, const __grid_constant__ NearMaps maps) {
  using Tin = __nv_bfloat16;
  constexpr int C16 = D / 8;  // 16-byte chunks of one head row
  const int h = blockIdx.x % p.nq, seg = blockIdx.x / p.nq;  // query head, segment of tiles
  const int s = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  extern __shared__ __align__(128) unsigned char smb_raw[];
  // 128-byte aligned base (the plan leaves 128 bytes of slack)
  unsigned char* smb = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smb_raw) + 127) & ~static_cast<uintptr_t>(127));
  const NearPlan& np = p.near;
  __shared__ __align__(8) uint64_t s_bar;
  __shared__ __align__(8) uint64_t s_ld[2];  // tensor copies of a stage landed
  __shared__ uint32_t s_tmem;
  __shared__ int s_ok;
  __shared__ long long s_pos;
  __shared__ __align__(16) float s_s0[2][128];  // S at the tile start, per stage
  __shared__ float s_gpow[kTile + 1];  // gamma_far^m

  pdl_trigger();
  pdl_wait();  // far state at the tile starts from far_carry_kernel
  unsigned char* blk = stream_block(p, s);
  if (tid <= kTile) s_gpow[tid] = powf(p.gamma_far, static_cast<float>(tid));
  if (tid == 0) {
    s_ok = header_matches(p);
    s_pos = reinterpret_cast<const long long*>(p.ws + p.ws_pos)[s];
    mbar_init(&s_bar, 1);
    mbar_init(&s_ld[0], 1);
    mbar_init(&s_ld[1], 1);
    mbar_fence_init();
  }
  __syncthreads();
  if (!s_ok) return;  // latched by far_agg_kernel
  if (warp == 0) tmem_alloc(&s_tmem, kTmemNear);
  const long long pos0 = s_pos;
  const long long ns = stream_len(p, s);  // tokens of this stream in the call
  const int K = p.K, nkv = p.nkv, g = h / p.G;
  const Tin* win_k = reinterpret_cast<const Tin*>(blk + p.so.win_k);
  const Tin* win_v = reinterpret_cast<const Tin*>(blk + p.so.win_v);
  const float* sst = reinterpret_cast<const float*>(p.ws + p.ws_sst) +
                     static_cast<long long>(s) * p.tiles_per_stream * nkv * D + g * D;
  const long long in_row0 = static_cast<long long>(s) * p.n;
  const Tin* kin = static_cast<const Tin*>(p.k) + in_row0 * nkv * D;
  const Tin* vin = static_cast<const Tin*>(p.v) + in_row0 * nkv * D;
  auto krow_g = [&](long long j) -> const Tin* {
    return j >= pos0 ? kin + ((j - pos0) * nkv + g) * D : win_k + ((j % K) * nkv + g) * D;
  };
  auto vrow_g = [&](long long j) -> const Tin* {
    return j >= pos0 ? vin + ((j - pos0) * nkv + g) * D : win_v + ((j % K) * nkv + g) * D;
  };
  unsigned char* pa_hi = smb + np.pa;
  unsigned char* pa_lo = pa_hi + kTile * kNS * 2;
  unsigned char* ga_hi = smb + np.ga;
  unsigned char* ga_lo = ga_hi + kTile * kNS * 2;
  for (int i = tid; i < 2 * kTile * kNS * 2 / 16; i += NT)  // P columns outside the bands stay zero
    reinterpret_cast<uint4*>(pa_hi)[i] = make_uint4(0u, 0u, 0u, 0u);
  const float gf = p.gamma_far, af = p.alpha_far;
  // G for the tiles whose first evicting token is r_ev (0 once t0 >= k).
  auto build_g = [&](int r_ev) {
    for (int i = tid; i < kTile * kNS; i += NT) {
      const int r = i / kNS, c = i % kNS;
      const int j = c - 16 + K;  // token whose evicted key is span row c
      float gv = 0.f;
      if (j >= r_ev && j <= r) gv = af * (1.0f - gf) * s_gpow[r - j];
      __nv_bfloat16 hb, lb;
      split_bf16(gv, hb, lb);
      const int off = blk_off(r, c);
      *reinterpret_cast<__nv_bfloat16*>(ga_hi + off) = hb;
      *reinterpret_cast<__nv_bfloat16*>(ga_lo + off) = lb;
    }
  };
  __syncthreads();  // s_gpow
  int g_built = -1;

  // Copies of tile i into stage st by the tensor-copy engine: D/8 boxes of
  // [64 tokens x 8 dims] for the queries and of [kNS rows x 8 dims] for the
  // key and value span (positions t0-16 .. t0+63), each landing as one
  // column of core matrices.  Token rows count over all streams of the
  // call, so rows past the stream hold another stream's inputs (finite,
  // masked out) and rows past the call read as zero; the first tile's rows
  // before the call are replaced from the state window (fix_history).
  constexpr unsigned kTileBytes = static_cast<unsigned>((D / 8) * (kTile + 2 * kNS) * 16);
  const int row0 = static_cast<int>(static_cast<long long>(s) * p.n);  // first token row of the stream
  auto issue = [&](int i, int st) {
    unsigned char* qa = smb + np.q[st];
    unsigned char* kb = smb + np.k[st];
    unsigned char* vb = smb + np.v[st];
    if (tid < D / 4) cp_async16(&s_s0[st][4 * tid], sst + static_cast<long long>(i) * nkv * D + 4 * tid);
    cp_async_commit();
    if (tid == 0) {
      const int rq = row0 + i * kTile, rkv = rq - 16;
      mbar_arrive_expect_tx(&s_ld[st], kTileBytes);
#pragma unroll
      for (int u = 0; u < D / 8; ++u) {
        tma_load_3d(qa + u * 1024, &maps.q, 8 * u, h, rq, &s_ld[st]);
        tma_load_3d(kb + u * kDStr, &maps.k, 8 * u, g, rkv, &s_ld[st]);
        tma_load_3d(vb + u * kDStr, &maps.v, 8 * u, g, rkv, &s_ld[st]);
      }
    }
  };
  // Span rows 0..15 of the call's first tile: positions before the call
  // from the state window, before position 0 zero.
  auto fix_history = [&](int st) {
    unsigned char* kb = smb + np.k[st];
    unsigned char* vb = smb + np.v[st];
    for (int c = tid; c < 16 * C16; c += NT) {
      const int r = c / C16, u = c % C16;
      const long long j = pos0 - 16 + r;
      const int off = kv_off(r, 8 * u);
      uint4 kv = make_uint4(0u, 0u, 0u, 0u), vv = kv;
      if (j >= 0) {
        kv = *reinterpret_cast<const uint4*>(krow_g(j) + 8 * u);
        vv = *reinterpret_cast<const uint4*>(vrow_g(j) + 8 * u);
      }
      *reinterpret_cast<uint4*>(kb + off) = kv;
      *reinterpret_cast<uint4*>(vb + off) = vv;
    }
  };

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  const uint32_t idesc_qk = umma_idesc_bf16(kTile, kNS, false);
  const uint32_t idesc_pv = umma_idesc_bf16(kTile, D, true);
  // this CTA's tiles (a ragged stream may end before them)
  const int tiles_s = static_cast<int>((ns + kTile - 1) / kTile);
  const int i0 = seg * p.tps, tiles = min(min(p.tiles_per_stream, tiles_s), i0 + p.tps);
  unsigned par = 0;
  bool ok = true;
  if (i0 < tiles) issue(i0, 0);
  for (int i = i0; i < tiles; ++i) {
    const int st = (np.stages == 2) ? ((i - i0) & 1) : 0;
    const unsigned ld_par = static_cast<unsigned>(((np.stages == 2) ? ((i - i0) >> 1) : (i - i0)) & 1);
    if (np.stages == 2 && i + 1 < tiles) {
      issue(i + 1, st ^ 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    if (!mbar_wait_bounded(&s_ld[st], ld_par, kMbarPollLimit, p.err)) ok = false;
    if (i == 0) fix_history(st);  // the call's first tile (the copies above have landed)
    const long long t0 = pos0 + static_cast<long long>(i) * kTile;
    const int Tt = static_cast<int>(min(static_cast<long long>(kTile), ns - static_cast<long long>(i) * kTile));
    const int r_ev = static_cast<int>(max(0LL, min(static_cast<long long>(Tt), K - t0)));
    if (r_ev != g_built) {  // uniform: the first tile of a stream start, then once more
      build_g(r_ev);
      g_built = r_ev;
    }
    fence_proxy_async_smem();  // copies, zero fills and G seen by the MMAs
    __syncthreads();
    const unsigned char* qa = smb + np.q[st];
    const unsigned char* kb = smb + np.k[st];
    const unsigned char* vb = smb + np.v[st];
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int k2 = 0; k2 < D / 16; ++k2)
        umma_bf16(tmem, umma_desc(qa + k2 * 2048, 1024, 128), umma_desc(kb + 2 * k2 * kDStr, kDStr, 128),
                  idesc_qk, k2 > 0);
      umma_commit(&s_bar);
    }
    if (!mbar_wait_bounded(&s_bar, par, kMbarPollLimit, p.err)) ok = false;
    par ^= 1u;
    tc_fence_after();
    // Band softmax: warp sp (< 4) holds rows 16 sp .. 16 sp + 15 in lanes
    // 0 .. 15, whose bands lie in span columns 16 sp .. 16 sp + 31.
    if (warp < 4) {
      const int sp = warp;
      float v[32];
      tmem_ld32(tmem + (static_cast<uint32_t>(32 * sp) << 16) + 16 * sp, v);
      if (lane < 16) {
        const int r = 16 * sp + lane;
        const int cmin = t0 < 16 ? static_cast<int>(16 - t0) : 0;  // first row at position >= 0
        float mx = -INFINITY;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int c = 16 * sp + j;
          const bool in = c >= r + 17 - K && c <= r + 16 && c >= cmin;
          v[j] = in ? v[j] * p.score_scale : -INFINITY;
          mx = fmaxf(mx, v[j]);
        }
        float sum = 0.f;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          v[j] = __expf(v[j] - mx);  // 0 outside the band
          sum += v[j];
        }
        const float inv = 1.f / sum;
#pragma unroll
        for (int g8 = 0; g8 < 4; ++g8) {
          uint32_t hw[4], lw[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            __nv_bfloat16 h0b, l0b, h1b, l1b;
            split_bf16(v[8 * g8 + 2 * e] * inv, h0b, l0b);
            split_bf16(v[8 * g8 + 2 * e + 1] * inv, h1b, l1b);
            hw[e] = static_cast<uint32_t>(__bfloat16_as_ushort(h0b)) |
                    (static_cast<uint32_t>(__bfloat16_as_ushort(h1b)) << 16);
            lw[e] = static_cast<uint32_t>(__bfloat16_as_ushort(l0b)) |
                    (static_cast<uint32_t>(__bfloat16_as_ushort(l1b)) << 16);
          }
          const int off = blk_off(r, 16 * sp + 8 * g8);
          *reinterpret_cast<uint4*>(pa_hi + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
          *reinterpret_cast<uint4*>(pa_lo + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
        }
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int k2 = 0; k2 < kNS / 16; ++k2) {
        const uint64_t bv = umma_desc(vb + k2 * 256, 128, kDStr);
        const uint64_t bk = umma_desc(kb + k2 * 256, 128, kDStr);
        umma_bf16(tmem + kTmemO, umma_desc(pa_hi + k2 * 2048, 1024, 128), bv, idesc_pv, k2 > 0);
        umma_bf16(tmem + kTmemO, umma_desc(pa_lo + k2 * 2048, 1024, 128), bv, idesc_pv, true);
        umma_bf16(tmem + kTmemO, umma_desc(ga_hi + k2 * 2048, 1024, 128), bk, idesc_pv, true);
        umma_bf16(tmem + kTmemO, umma_desc(ga_lo + k2 * 2048, 1024, 128), bk, idesc_pv, true);
      }
      umma_commit(&s_bar);
    }
    if (!mbar_wait_bounded(&s_bar, par, kMbarPollLimit, p.err)) ok = false;
    par ^= 1u;
    tc_fence_after();
    {  // x = X + alpha_far gamma^m(r) S0 into out: warp w takes rows 16 (w%4) ..,
       // half the head dims
      const int sp = warp & 3, colh = (warp >> 2) * (D / 2);
      const int r = 16 * sp + lane;
      const float c0s = af * s_gpow[min(kTile, max(0, r - r_ev + 1))];
      float* orow = p.out + (in_row0 + (t0 - pos0) + r) * p.H + h * D + colh;
#pragma unroll
      for (int c0 = 0; c0 < D / 2; c0 += 32) {
        float v[32];
        tmem_ld32(tmem + (static_cast<uint32_t>(32 * sp) << 16) + kTmemO + colh + c0, v);
        if (lane < 16 && r < Tt && ok) {
          const float* s0 = s_s0[st] + colh + c0;
#pragma unroll
          for (int j = 0; j < 32; j += 4)
            *reinterpret_cast<float4*>(orow + c0 + j) =
                make_float4(fmaf(c0s, s0[j], v[j]), fmaf(c0s, s0[j + 1], v[j + 1]),
                            fmaf(c0s, s0[j + 2], v[j + 2]), fmaf(c0s, s0[j + 3], v[j + 3]));
        }
      }
    }
    tc_fence_before();
    __syncthreads();  // stage, P and accumulators free again
    if (np.stages != 2 && i + 1 < tiles) issue(i + 1, 0);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemNear);
  }
}

// ======================================================================
// 1+2. fused: near field, far field, x, pool scores and field aggregates
// ======================================================================
// One CTA per (stream, segment of consecutive tiles) walks its tiles and,
// per tile, every query head h (step j = tile * n_q + h).  Per step, on the
// tcgen05 tensor cores with fp32 accumulators in tensor memory:
//   QK(j):   scores[64 x 80] = Q_h . K_span^T, the band softmax on warps 2-5
//            [P1 §2.1 eq. O_near];
//   PV(j):   X_h[64 x D] = P . V_span + G . K_span (hi and lo of P and of
//            the far-field weights G, as in near_tc_kernel); warps 6-9 add
//            alpha_far gamma^m S_start [P1 §2.1 eq. O], store x (fp32) for
//            the output kernel and split it into bf16 hi/lo blocks;
//   POOL(j): pool[64 x 64 slots] += X_h . slot_h^T (hi*hi + hi*lo + lo*hi)
//            over the heads of the tile [P3 §2.1 channel 3], and the EMA
//            field over the tile from zero for the head's columns,
//            A[c] = sum_r (1-g) g^(Tt-1-r) x[r][c] [P3 §2.1 channel 2], as
//            the transposed product X_h^T . F with the weights in column 0
//            of F (column 1: the stream's last tile when it is short).
// After a tile's last head its scores, |x|^2 per token and the slot norms
// give softmax(cos/T); the weights go to the workspace as split bf16 blocks,
// as pool_kernel writes them, and x, the field aggregates and the output
// segments' halo rows as near_tc_kernel and pool_kernel write them: the
// output kernel is the same.
//
// Warp roles (one elected lane issues): warp 0 loads (tensor copies of q per
// head and of the key/value span per KV head), warp 14 the bulk copies of
// each head's slot blocks; warp 1 issues the MMAs, for step j QK(j), PV(j-1) and
// POOL(j-2); warps 2-5 run the band softmax and the tile's pool softmax;
// warps 6-13 the x epilogue, two per lane quarter of the accumulator, each
// on half of the head's columns.  Scores
// and X accumulators are double-buffered in tensor memory, queries and slot
// blocks double-buffered in shared memory; every hand-off is an mbarrier
// with a bounded wait.
constexpr int NTF = 480;              // threads of the fused kernel: 15 warps
constexpr int kEpiWarps = 8;          // x epilogue warps (warps 6 .. 13)
constexpr int kFusedWarps = NTF / 32;  // the last one loads slot blocks
constexpr int kTmemFused = 512;       // all of an SM's tensor memory: one CTA per SM
constexpr int kFColS = 0;             // [2] band scores, kNS columns each
constexpr int kFColPool = 2 * kNS;    // pool scores, 64 columns
constexpr int kFColFagg = kFColPool + kSlots;  // field aggregates, 16 columns
constexpr int kFColX = 256;           // [2] X accumulators, D columns each
static_assert(kFColFagg + 16 <= kFColX, "tensor-memory columns of the fused kernel");

template <int D>
struct FusedPlan {
  static constexpr int kvb = (D / 8) * kDStr;             // key (or value) span block
  static constexpr int qb = kTile * D * 2;                // one head's queries
  static constexpr int slb = (D / kBlk) * 2 * kBlkBytes;  // one head's slot blocks (hi, lo per chunk)
  static constexpr int pb = kTile * kNS * 2;              // a P or G block (hi or lo)
  static constexpr int xb = kTile * D * 2;                // an X block (hi or lo)
  static constexpr int kk = 1024;                         // mbarriers before it
  static constexpr int vv = kk + kvb;
  static constexpr int q0 = vv + kvb;                     // [2]
  static constexpr int sl0 = q0 + 2 * qb;                 // [2]
  static constexpr int pa = sl0 + 2 * slb;                // hi, lo
  static constexpr int ga = pa + 2 * pb;                  // hi, lo
  static constexpr int xa = ga + 2 * pb;                  // hi, lo
  static constexpr int fa = xa + 2 * xb;                  // hi, lo [16 x 64] blocks of F
  static constexpr int total = fa + 2 * kBlk16Bytes + 128;  // 128: base alignment slack
};
static_assert(FusedPlan<128>::total <= 227 * 1024 - 2048, "fused kernel shared memory");

// barrier slots
enum : int {
  kFbKvFull = 0, kFbKvFix, kFbKvEmpty,
  kFbQFull, kFbQEmpty = kFbQFull + 2,
  kFbSlFull = kFbQEmpty + 2, kFbSlEmpty = kFbSlFull + 2,
  kFbSFull = kFbSlEmpty + 2, kFbSEmpty = kFbSFull + 2,
  kFbPFull = kFbSEmpty + 2, kFbPEmpty,
  kFbOFull, kFbOEmpty = kFbOFull + 2,
  kFbXFull = kFbOEmpty + 2, kFbXEmpty,
  kFbScFull, kFbScEmpty, kFbSqFull, kFbSqEmpty, kFbProbe,
  kFbCount
};
static_assert(kFbCount * 8 <= 1024, "fused kernel barriers");

template <int D>
__global__ void __launch_bounds__(NTF, 1)
fused_kernel(const __grid_constant__ PrefillParams p, const __grid_constant__ NearMaps maps) {
  using Tin = __nv_bfloat16;
  using FP = FusedPlan<D>;
  constexpr int C16 = D / 8;  // 16-byte chunks of one head row
  const int seg = blockIdx.x, s = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  extern __shared__ __align__(128) unsigned char smf_raw[];
  unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smf_raw) + 127) &
                                                       ~static_cast<uintptr_t>(127));
  uint64_t* bar = reinterpret_cast<uint64_t*>(sm);
  __shared__ uint32_t s_tmem;
  __shared__ int s_ok;
  __shared__ long long s_pos;
  __shared__ float s_gpow[kTile + 1];  // gamma_far^m
  __shared__ float s_norm[kSlots];     // slot norms of the layer
  __shared__ float s_sq[2][kTile];     // |x|^2 per token of the tile being finished, per column half
  __shared__ __align__(16) float s_s0[128];  // S at the tile start of the epilogue's KV head

  pdl_trigger();
  pdl_wait();  // far state at the tile starts from far_carry_kernel
  const int l = p.l0 + s / p.B;
  if (tid <= kTile) s_gpow[tid] = powf(p.gamma_far, static_cast<float>(tid));
  if (tid < kSlots) s_norm[tid] = p.slot_norm[static_cast<size_t>(l) * kSlots + tid];
  if (tid == 0) {
    s_ok = header_matches(p);
    s_pos = reinterpret_cast<const long long*>(p.ws + p.ws_pos)[s];
    for (int b = 0; b < kFbCount; ++b) {
      int count = 1;
      if (b == kFbSEmpty || b == kFbSEmpty + 1 || b == kFbPFull || b == kFbScEmpty || b == kFbSqEmpty)
        count = 4;  // one arrival per softmax warp
      if (b == kFbOEmpty || b == kFbOEmpty + 1 || b == kFbXFull || b == kFbSqFull)
        count = kEpiWarps;  // one arrival per epilogue warp
      mbar_init(bar + b, count);
    }
    mbar_fence_init();
  }
  __syncthreads();
  if (!s_ok) return;  // latched by far_agg_kernel
  const long long pos0 = s_pos;
  const long long ns = stream_len(p, s);  // tokens of this stream in the call
  const int tiles_s = static_cast<int>((ns + kTile - 1) / kTile);
  const int i0 = seg * p.tps, i1 = min(min(p.tiles_per_stream, tiles_s), i0 + p.tps);
  if (i0 >= i1) return;  // past a ragged stream's end
  const int nq = p.nq, G = p.G, nkv = p.nkv, K = p.K;
  const int nsteps = (i1 - i0) * nq;
  if (warp == 1) tmem_alloc(&s_tmem, kTmemFused);  // one CTA per SM (shared memory): never waits long

  unsigned char* kk = sm + FP::kk;
  unsigned char* vv = sm + FP::vv;
  unsigned char* pa_hi = sm + FP::pa;
  unsigned char* pa_lo = pa_hi + FP::pb;
  unsigned char* ga_hi = sm + FP::ga;
  unsigned char* ga_lo = ga_hi + FP::pb;
  unsigned char* xa_hi = sm + FP::xa;
  unsigned char* xa_lo = xa_hi + FP::xb;
  unsigned char* fa_hi = sm + FP::fa;
  unsigned char* fa_lo = fa_hi + kBlk16Bytes;
  const float gf = p.gamma_far, af = p.alpha_far, ge = p.ema_gamma;
  // P columns outside the bands stay zero; G for every tile (the rows a
  // tile's first tokens would evict before position k multiply span rows
  // before position 0, which are zero); F: column 0 the field weights of a
  // full tile, column 1 those of the stream's last tile if it is short.
  for (int i = tid; i < 2 * FP::pb / 16; i += NTF) reinterpret_cast<uint4*>(pa_hi)[i] = make_uint4(0u, 0u, 0u, 0u);
  for (int i = tid; i < kTile * kNS; i += NTF) {
    const int r = i / kNS, c = i % kNS;
    const int j = c - 16 + K;  // token whose evicted key is span row c
    const float gv = (j >= 0 && j <= r) ? af * (1.0f - gf) * powf(gf, static_cast<float>(r - j)) : 0.f;
    __nv_bfloat16 hb, lb;
    split_bf16(gv, hb, lb);
    const int off = blk_off(r, c);
    *reinterpret_cast<__nv_bfloat16*>(ga_hi + off) = hb;
    *reinterpret_cast<__nv_bfloat16*>(ga_lo + off) = lb;
  }
  const int t_last = static_cast<int>(ns - static_cast<long long>(tiles_s - 1) * kTile);  // tokens of the last tile
  for (int i = tid; i < 16 * kTile; i += NTF) {
    const int n = i / kTile, r = i % kTile;
    float fv = 0.f;
    if (n == 0) fv = (1.0f - ge) * powf(ge, static_cast<float>(kTile - 1 - r));
    if (n == 1 && r < t_last) fv = (1.0f - ge) * powf(ge, static_cast<float>(t_last - 1 - r));
    __nv_bfloat16 hb, lb;
    split_bf16(fv, hb, lb);
    const int off = blk16_off(n, r);
    *reinterpret_cast<__nv_bfloat16*>(fa_hi + off) = hb;
    *reinterpret_cast<__nv_bfloat16*>(fa_lo + off) = lb;
  }
  fence_proxy_async_smem();  // zero fills, G and F seen by the MMAs
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  const int row0 = static_cast<int>(static_cast<long long>(s) * p.n);  // first token row of the stream
  const long long in_row0 = static_cast<long long>(s) * p.n;
  bool ok = true;
  auto wait = [&](int b, unsigned parity) {
    if (!mbar_wait_bounded(bar + b, parity, kMbarPollLimit, p.err)) ok = false;
  };
  auto tile_rows = [&](int i) -> int {
    return static_cast<int>(min(static_cast<long long>(kTile), ns - static_cast<long long>(i) * kTile));
  };

  if (warp == 0) {
    // ---- loads ------------------------------------------------------------
    unsigned char* blk = stream_block(p, s);
    const Tin* win_k = reinterpret_cast<const Tin*>(blk + p.so.win_k);
    const Tin* win_v = reinterpret_cast<const Tin*>(blk + p.so.win_v);
    constexpr unsigned kKvBytes = static_cast<unsigned>(2 * C16 * kNS * 16);
    int kvc = 0;  // span copies issued
    for (int j = 0; j < nsteps; ++j) {
      const int h = j % nq, i = i0 + j / nq, g = h / G, b = j & 1;
      if (h % G == 0) {
        if (lane == 0) {
          if (kvc > 0) wait(kFbKvEmpty, static_cast<unsigned>((kvc - 1) & 1));
          mbar_arrive_expect_tx(bar + kFbKvFull, kKvBytes);
          const int rkv = row0 + i * kTile - 16;
#pragma unroll
          for (int u = 0; u < C16; ++u) {
            tma_load_3d(kk + u * kDStr, &maps.k, 8 * u, g, rkv, bar + kFbKvFull);
            tma_load_3d(vv + u * kDStr, &maps.v, 8 * u, g, rkv, bar + kFbKvFull);
          }
        }
        if (i == 0) {
          // span rows 0..15 of the call's first tile: positions before the
          // call from the state window, before position 0 zero
          if (lane == 0) wait(kFbKvFull, static_cast<unsigned>(kvc & 1));
          __syncwarp();
          for (int c = lane; c < 16 * C16; c += 32) {
            const int r = c / C16, u = c % C16;
            const long long jp = pos0 - 16 + r;
            uint4 kv4 = make_uint4(0u, 0u, 0u, 0u), vv4 = kv4;
            if (jp >= 0) {
              kv4 = *reinterpret_cast<const uint4*>(win_k + ((jp % K) * nkv + g) * D + 8 * u);
              vv4 = *reinterpret_cast<const uint4*>(win_v + ((jp % K) * nkv + g) * D + 8 * u);
            }
            *reinterpret_cast<uint4*>(kk + kv_off(r, 8 * u)) = kv4;
            *reinterpret_cast<uint4*>(vv + kv_off(r, 8 * u)) = vv4;
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar + kFbKvFix);
        }
        ++kvc;
      }
      if (lane == 0) {
        if (j >= 2) wait(kFbQEmpty + b, static_cast<unsigned>(((j >> 1) - 1) & 1));
        unsigned char* qa = sm + FP::q0 + b * FP::qb;
        mbar_arrive_expect_tx(bar + kFbQFull + b, static_cast<unsigned>(FP::qb));
#pragma unroll
        for (int u = 0; u < C16; ++u) tma_load_3d(qa + u * 1024, &maps.q, 8 * u, h, row0 + i * kTile, bar + kFbQFull + b);
      }
    }
  } else if (warp == kFusedWarps - 1) {
    // ---- slot blocks of each head (a warp of their own: their stage frees
    // only when the head's pool MMAs complete) ------------------------------------
    if (lane == 0) {
      const unsigned char* img_l = p.slot_img + static_cast<size_t>(l) * (p.H / kBlk) * 2 * kBlkBytes;
      for (int j = 0; j < nsteps; ++j) {
        const int h = j % nq, b = j & 1;
        if (j >= 2) wait(kFbSlEmpty + b, static_cast<unsigned>(((j >> 1) - 1) & 1));
        mbar_arrive_expect_tx(bar + kFbSlFull + b, static_cast<unsigned>(FP::slb));
        bulk_g2s(sm + FP::sl0 + b * FP::slb, img_l + static_cast<size_t>(h) * FP::slb, static_cast<unsigned>(FP::slb),
                 bar + kFbSlFull + b);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---- MMAs ---------------------------------------------------------------
    if (lane == 0) {
      const uint32_t idesc_qk = umma_idesc_bf16(kTile, kNS, false);
      const uint32_t idesc_pv = umma_idesc_bf16(kTile, D, true);
      const uint32_t idesc_sc = umma_idesc_bf16(kTile, kSlots, false);
      const uint32_t idesc_fa = umma_idesc_bf16_ab(D, 16, true, false);  // X^T (MN-major) . F
      int kvw = 0;  // span copies waited for
      auto do_qk = [&](int j) {
        const int h = j % nq, i = i0 + j / nq, b = j & 1;
        if (h % G == 0) {
          wait(kFbKvFull, static_cast<unsigned>(kvw & 1));
          if (i == 0) wait(kFbKvFix, static_cast<unsigned>(kvw & 1));  // kvw = KV head here
          ++kvw;
        }
        wait(kFbQFull + b, static_cast<unsigned>((j >> 1) & 1));
        if (j >= 2) wait(kFbSEmpty + b, static_cast<unsigned>(((j >> 1) - 1) & 1));
        tc_fence_after();
        const unsigned char* qa = sm + FP::q0 + b * FP::qb;
#pragma unroll
        for (int k2 = 0; k2 < D / 16; ++k2)
          umma_bf16(tmem + kFColS + b * kNS, umma_desc(qa + k2 * 2048, 1024, 128),
                    umma_desc(kk + 2 * k2 * kDStr, kDStr, 128), idesc_qk, k2 > 0);
        umma_commit(bar + kFbSFull + b);
        umma_commit(bar + kFbQEmpty + b);
      };
      auto do_pv = [&](int j) {
        const int h = j % nq, b = j & 1;
        wait(kFbPFull, static_cast<unsigned>(j & 1));
        if (j >= 2) wait(kFbOEmpty + b, static_cast<unsigned>(((j >> 1) - 1) & 1));
        tc_fence_after();
        const uint32_t dst = tmem + kFColX + b * D;
#pragma unroll
        for (int k2 = 0; k2 < kNS / 16; ++k2) {
          const uint64_t bv = umma_desc(vv + k2 * 256, 128, kDStr);
          const uint64_t bk = umma_desc(kk + k2 * 256, 128, kDStr);
          umma_bf16(dst, umma_desc(pa_hi + k2 * 2048, 1024, 128), bv, idesc_pv, k2 > 0);
          umma_bf16(dst, umma_desc(pa_lo + k2 * 2048, 1024, 128), bv, idesc_pv, true);
          umma_bf16(dst, umma_desc(ga_hi + k2 * 2048, 1024, 128), bk, idesc_pv, true);
          umma_bf16(dst, umma_desc(ga_lo + k2 * 2048, 1024, 128), bk, idesc_pv, true);
        }
        umma_commit(bar + kFbOFull + b);
        umma_commit(bar + kFbPEmpty);
        if (h % G == G - 1 || j == nsteps - 1) umma_commit(bar + kFbKvEmpty);  // span no longer read
      };
      auto do_pool = [&](int j) {
        const int h = j % nq, ti = j / nq, b = j & 1;
        wait(kFbXFull, static_cast<unsigned>(j & 1));
        wait(kFbSlFull + b, static_cast<unsigned>((j >> 1) & 1));
        if (h == 0 && ti >= 1) wait(kFbScEmpty, static_cast<unsigned>((ti - 1) & 1));
        tc_fence_after();
        const unsigned char* sl = sm + FP::sl0 + b * FP::slb;
#pragma unroll
        for (int c = 0; c < D / kBlk; ++c) {
          const unsigned char* shi = sl + c * 2 * kBlkBytes;
          const unsigned char* slo = shi + kBlkBytes;
#pragma unroll
          for (int k = 0; k < kBlk / 16; ++k) {
            const uint64_t ah = umma_desc(xa_hi + c * kBlkBytes + k * 2048, 1024, 128);
            const uint64_t al = umma_desc(xa_lo + c * kBlkBytes + k * 2048, 1024, 128);
            const uint64_t bh = umma_desc(shi + k * 2048, 1024, 128), bl = umma_desc(slo + k * 2048, 1024, 128);
            umma_bf16(tmem + kFColPool, ah, bh, idesc_sc, h > 0 || c > 0 || k > 0);
            umma_bf16(tmem + kFColPool, ah, bl, idesc_sc, true);
            umma_bf16(tmem + kFColPool, al, bh, idesc_sc, true);
          }
        }
#pragma unroll
        for (int k = 0; k < kTile / 16; ++k) {
          const uint64_t ah = umma_desc(xa_hi + k * 256, 128, 1024), al = umma_desc(xa_lo + k * 256, 128, 1024);
          const uint64_t bh = umma_desc(fa_hi + k * 512, 256, 128), bl = umma_desc(fa_lo + k * 512, 256, 128);
          umma_bf16(tmem + kFColFagg, ah, bh, idesc_fa, k > 0);
          umma_bf16(tmem + kFColFagg, ah, bl, idesc_fa, true);
          umma_bf16(tmem + kFColFagg, al, bh, idesc_fa, true);
        }
        umma_commit(bar + kFbXEmpty);
        umma_commit(bar + kFbSlEmpty + b);
        if (h == nq - 1) umma_commit(bar + kFbScFull);
      };
      // Step j: QK(j), PV(j-1), POOL(j-2); PV first where step j opens a
      // KV head's span, whose copy waits for the last PV on the previous one.
      for (int j = 0; j <= nsteps + 1; ++j) {
        if (j < nsteps && (j % nq) % G == 0) {
          if (j >= 1) do_pv(j - 1);
          do_qk(j);
        } else {
          if (j < nsteps) do_qk(j);
          if (j >= 1 && j <= nsteps) do_pv(j - 1);
        }
        if (j >= 2) do_pool(j - 2);
      }
    }
    __syncwarp();
  } else if (warp < 6) {
    // ---- band softmax; the tile's pool softmax -------------------------------
    const int qd = warp & 3;  // lane quarter: rows 16 qd .. 16 qd + 15 in lanes 0..15
    const int r = 16 * qd + lane;
    const uint32_t lane_base = static_cast<uint32_t>(32 * qd) << 16;
    auto finish = [&](int ti) {
      const int i = i0 + ti;
      const int Tt = tile_rows(i);
      wait(kFbScFull, static_cast<unsigned>(ti & 1));
      wait(kFbSqFull, static_cast<unsigned>(ti & 1));
      tc_fence_after();
      float sv[kSlots];
      tmem_ld32(tmem + lane_base + kFColPool, *reinterpret_cast<float(*)[32]>(sv));
      tmem_ld32(tmem + lane_base + kFColPool + 32, *reinterpret_cast<float(*)[32]>(sv + 32));
      const float sq = lane < 16 ? s_sq[0][r] + s_sq[1][r] : 0.f;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(bar + kFbScEmpty);
        mbar_arrive(bar + kFbSqEmpty);
      }
      // Test hook: a bounded wait on a barrier that nothing completes.
      if (tid == 64 && static_cast<long long>(i) * p.n_streams + s == p.withhold_tile) {
        mbar_arrive_expect_tx(bar + kFbProbe, 16u);
        mbar_wait_bounded(bar + kFbProbe, 0, p.spin_limit, p.err);
      }
      if (lane < 16) {
        // softmax(cos/T) per token [P3 §2.1 channel 3]; rows past the tile
        // get zero weights
        const float nx = fmaxf(sqrtf(sq), kNormFloor);
        float mx = -INFINITY;
#pragma unroll
        for (int e = 0; e < kSlots; ++e) {
          sv[e] = sv[e] / (nx * s_norm[e]) * p.inv_temp;
          mx = fmaxf(mx, sv[e]);
        }
        float sum = 0.f;
#pragma unroll
        for (int e = 0; e < kSlots; ++e) {
          sv[e] = expf(sv[e] - mx);
          sum += sv[e];
        }
        const float inv = r < Tt ? 1.f / sum : 0.f;
        unsigned char* wblk = p.ws + p.ws_w + (static_cast<long long>(s) * p.tiles_per_stream + i) * 2 * kBlkBytes;
#pragma unroll
        for (int g8 = 0; g8 < kSlots / 8; ++g8) {
          uint32_t hw[4], lw[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            __nv_bfloat16 h0b, l0b, h1b, l1b;
            split_bf16(sv[8 * g8 + 2 * e] * inv, h0b, l0b);
            split_bf16(sv[8 * g8 + 2 * e + 1] * inv, h1b, l1b);
            hw[e] = static_cast<uint32_t>(__bfloat16_as_ushort(h0b)) |
                    (static_cast<uint32_t>(__bfloat16_as_ushort(h1b)) << 16);
            lw[e] = static_cast<uint32_t>(__bfloat16_as_ushort(l0b)) |
                    (static_cast<uint32_t>(__bfloat16_as_ushort(l1b)) << 16);
          }
          if (ok) {
            const int off = blk_off(r, 8 * g8);
            *reinterpret_cast<uint4*>(wblk + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
            *reinterpret_cast<uint4*>(wblk + kBlkBytes + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
          }
        }
      }
    };
    for (int j = 0; j < nsteps; ++j) {
      const int ti = j / nq, b = j & 1;
      const long long t0 = pos0 + static_cast<long long>(i0 + ti) * kTile;
      wait(kFbSFull + b, static_cast<unsigned>((j >> 1) & 1));
      tc_fence_after();
      float v[32];
      tmem_ld32(tmem + lane_base + kFColS + b * kNS + 16 * qd, v);  // the band of rows 16 qd .. lies in span columns 16 qd .. 16 qd + 31
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar + kFbSEmpty + b);
      uint32_t hw[4][4], lw[4][4];
      {
        const int cmin = t0 < 16 ? static_cast<int>(16 - t0) : 0;  // first span row at position >= 0
        float mx = -INFINITY;
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const int c = 16 * qd + e;
          const bool in = c >= r + 17 - K && c <= r + 16 && c >= cmin;
          v[e] = in ? v[e] * p.score_scale : -INFINITY;
          mx = fmaxf(mx, v[e]);
        }
        float sum = 0.f;
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          v[e] = __expf(v[e] - mx);  // 0 outside the band
          sum += v[e];
        }
        const float inv = 1.f / sum;
#pragma unroll
        for (int g8 = 0; g8 < 4; ++g8)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            __nv_bfloat16 h0b, l0b, h1b, l1b;
            split_bf16(v[8 * g8 + 2 * e] * inv, h0b, l0b);
            split_bf16(v[8 * g8 + 2 * e + 1] * inv, h1b, l1b);
            hw[g8][e] = static_cast<uint32_t>(__bfloat16_as_ushort(h0b)) |
                        (static_cast<uint32_t>(__bfloat16_as_ushort(h1b)) << 16);
            lw[g8][e] = static_cast<uint32_t>(__bfloat16_as_ushort(l0b)) |
                        (static_cast<uint32_t>(__bfloat16_as_ushort(l1b)) << 16);
          }
      }
      if (j >= 1) wait(kFbPEmpty, static_cast<unsigned>((j - 1) & 1));  // PV(j-1) has read P
      if (lane < 16) {
#pragma unroll
        for (int g8 = 0; g8 < 4; ++g8) {
          const int off = blk_off(r, 16 * qd + 8 * g8);
          *reinterpret_cast<uint4*>(pa_hi + off) = make_uint4(hw[g8][0], hw[g8][1], hw[g8][2], hw[g8][3]);
          *reinterpret_cast<uint4*>(pa_lo + off) = make_uint4(lw[g8][0], lw[g8][1], lw[g8][2], lw[g8][3]);
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar + kFbPFull);
      if (j % nq == 0 && ti >= 1) finish(ti - 1);
    }
    finish((nsteps - 1) / nq);
  } else {
    // ---- x epilogue ------------------------------------------------------------
    const int qd = warp & 3;  // lane quarter: rows 16 qd .. 16 qd + 15 in lanes 0..15
    const int hf = (warp - 6) >> 2;  // column half of the head
    const int r = 16 * qd + lane;
    const uint32_t lane_base = static_cast<uint32_t>(32 * qd) << 16;
    const float* sst = reinterpret_cast<const float*>(p.ws + p.ws_sst) +
                       static_cast<long long>(s) * p.tiles_per_stream * nkv * D;
    float* fagg = reinterpret_cast<float*>(p.ws + p.ws_fagg) + static_cast<long long>(s) * p.tiles_per_stream * p.H;
    // field aggregate of step j's columns: column 0 of the accumulator for a
    // full tile, column 1 for a short last tile.  M = 128 (D = 128): column
    // c in lane c; M = 64: column c in lane (c % 16) + 32 (c / 16).
    auto store_fagg = [&](int j) {
      const int h = j % nq, i = i0 + j / nq;
      tc_fence_after();
      float fv[2];
      tmem_ld2(tmem + lane_base + kFColFagg, fv);
      const int c = D == 128 ? 32 * qd + lane : 16 * qd + lane;
      if (hf == 0 && (D == 128 || lane < 16) && ok)
        fagg[static_cast<long long>(i) * p.H + h * D + c] = tile_rows(i) == kTile ? fv[0] : fv[1];
    };
    float sq4[4] = {0.f, 0.f, 0.f, 0.f};  // |x|^2 of row r over the tile's heads so far (four partial sums)
    constexpr int NC = D / 64;             // 32-column chunks of this warp's half of a head
    for (int j = 0; j < nsteps; ++j) {
      const int h = j % nq, ti = j / nq, i = i0 + ti, g = h / G, b = j & 1;
      const long long t0 = pos0 + static_cast<long long>(i) * kTile;
      const int Tt = tile_rows(i);
      const int r_ev = static_cast<int>(max(0LL, min(static_cast<long long>(Tt), K - t0)));
      const float c0s = af * s_gpow[min(kTile, max(0, r - r_ev + 1))];
      if (h % G == 0) {  // the KV head's S at the tile start, staged once for the eight warps
        named_bar_sync(1, kEpiWarps * 32);  // every epilogue warp is done with the previous one
        for (int e = tid - 6 * 32; e < D; e += kEpiWarps * 32) s_s0[e] = sst[(static_cast<long long>(i) * nkv + g) * D + e];
        named_bar_sync(1, kEpiWarps * 32);
      }
      const bool live = lane < 16 && r < Tt && ok;
      float* orow = p.out + (in_row0 + static_cast<long long>(i) * kTile + r) * p.H + h * D;
      // the last kHalo rows of a tile that ends an output segment lead the next one
      const bool halo_row = r >= kTile - kHalo && (i + 1) % p.tps_out == 0 &&
                            (i + 1) * static_cast<long long>(kTile) < ns;
      float* hrow = reinterpret_cast<float*>(p.ws + p.ws_halo) +
                    ((static_cast<long long>(s) * p.nseg_out + (i + 1) / p.tps_out - 1) * kHalo +
                     (r - (kTile - kHalo))) * p.H + h * D;
      wait(kFbOFull + b, static_cast<unsigned>((j >> 1) & 1));
      tc_fence_after();
      float v[NC][32];
#pragma unroll
      for (int u = 0; u < NC; ++u) tmem_ld32(tmem + lane_base + kFColX + b * D + 32 * (hf * NC + u), v[u]);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar + kFbOEmpty + b);  // the accumulator is in registers
      // x = X + alpha_far gamma^m S_start [P1 §2.1 eq. O], stored for the output kernel
#pragma unroll
      for (int u = 0; u < NC; ++u) {
        const int c0 = 32 * (hf * NC + u);
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          const float4 sv4 = *reinterpret_cast<const float4*>(s_s0 + c0 + e);
          v[u][e] = r < Tt ? fmaf(c0s, sv4.x, v[u][e]) : 0.f;
          v[u][e + 1] = r < Tt ? fmaf(c0s, sv4.y, v[u][e + 1]) : 0.f;
          v[u][e + 2] = r < Tt ? fmaf(c0s, sv4.z, v[u][e + 2]) : 0.f;
          v[u][e + 3] = r < Tt ? fmaf(c0s, sv4.w, v[u][e + 3]) : 0.f;
          sq4[(e >> 2) & 3] = fmaf(v[u][e], v[u][e], fmaf(v[u][e + 1], v[u][e + 1],
                                   fmaf(v[u][e + 2], v[u][e + 2], fmaf(v[u][e + 3], v[u][e + 3], sq4[(e >> 2) & 3]))));
          if (live) {
            const float4 o4 = make_float4(v[u][e], v[u][e + 1], v[u][e + 2], v[u][e + 3]);
            *reinterpret_cast<float4*>(orow + c0 + e) = o4;
            if (halo_row) *reinterpret_cast<float4*>(hrow + c0 + e) = o4;
          }
        }
      }
      if (j >= 1) {  // POOL(j-1) has read X: its field aggregate is ready
        wait(kFbXEmpty, static_cast<unsigned>((j - 1) & 1));
        store_fagg(j - 1);
      }
      if (lane < 16) {
#pragma unroll
        for (int u = 0; u < NC; ++u)
#pragma unroll
          for (int g8 = 0; g8 < 4; ++g8) {
            uint32_t hw[4], lw[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              __nv_bfloat16 h0b, l0b, h1b, l1b;
              split_bf16(v[u][8 * g8 + 2 * e], h0b, l0b);
              split_bf16(v[u][8 * g8 + 2 * e + 1], h1b, l1b);
              hw[e] = static_cast<uint32_t>(__bfloat16_as_ushort(h0b)) |
                      (static_cast<uint32_t>(__bfloat16_as_ushort(h1b)) << 16);
              lw[e] = static_cast<uint32_t>(__bfloat16_as_ushort(l0b)) |
                      (static_cast<uint32_t>(__bfloat16_as_ushort(l1b)) << 16);
            }
            const int col = 32 * (hf * NC + u) + 8 * g8;  // X blocks: [64 x D], 8-column groups 1 KB apart
            const int off = (col >> 3) * 1024 + (r >> 3) * 128 + (r & 7) * 16;
            *reinterpret_cast<uint4*>(xa_hi + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
            *reinterpret_cast<uint4*>(xa_lo + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
          }
      }
      tc_fence_before();
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar + kFbXFull);
      if (h == nq - 1) {  // |x|^2 of the tile's tokens for its pool softmax
        if (ti >= 1) wait(kFbSqEmpty, static_cast<unsigned>((ti - 1) & 1));
        if (lane < 16) s_sq[hf][r] = (sq4[0] + sq4[1]) + (sq4[2] + sq4[3]);
#pragma unroll
        for (int e = 0; e < 4; ++e) sq4[e] = 0.f;
        __syncwarp();
        if (lane == 0) mbar_arrive(bar + kFbSqFull);
      }
    }
    wait(kFbXEmpty, static_cast<unsigned>((nsteps - 1) & 1));
    store_fagg(nsteps - 1);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemFused);
  }
}

// ======================================================================
// 2. pool scores and weights
// ======================================================================

// Shared-memory plan of pool_kernel (byte offsets).
struct PoolPlan {
  static constexpr int bars = 0;                        // 6 mbarriers
  static constexpr int tmem = 64;                       // tensor-memory address
  static constexpr int img = 128;                       // [3][hi, lo] slot blocks
  static constexpr int xsp = img + 3 * 2 * kBlkBytes;   // [2][hi, lo] split x blocks
  static constexpr int sc = xsp + 2 * 2 * kBlkBytes;    // [64][65] fp32 scores
  static constexpr int ss = sc + kTile * kScStride * 4; // [16][64] |x|^2 partials
  static constexpr int total = ss + 16 * kTile * 4;
};

__global__ void __launch_bounds__(NT, 2) pool_kernel(const PrefillParams p) {
  const int tile = blockIdx.x, s = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  extern __shared__ __align__(16) unsigned char smb[];
  uint64_t* bar_img = reinterpret_cast<uint64_t*>(smb + PoolPlan::bars);  // [3] slot blocks landed
  uint64_t* bar_mma = bar_img + 3;                                       // [2] MMAs of a split stage done
  uint64_t* bar_probe = bar_img + 5;                                     // test hook only
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smb + PoolPlan::tmem);
  float* sc = reinterpret_cast<float*>(smb + PoolPlan::sc);
  float* sqp = reinterpret_cast<float*>(smb + PoolPlan::ss);
  __shared__ int s_ok;
  __shared__ float ssq[kTile];

  pdl_trigger();
  pdl_wait();  // x is written by near_kernel
  if (tid == 0) {
    s_ok = header_matches(p);
    for (int b = 0; b < 6; ++b) mbar_init(bar_img + b, 1);
    mbar_fence_init();
  }
  __syncthreads();
  if (!s_ok || stream_len(p, s) <= static_cast<long long>(tile) * kTile) return;  // past a ragged stream's end
  if (warp == 0) tmem_alloc(tmem_slot, kTmemCols);
  const int l = p.l0 + s / p.B;
  const long long n0 = static_cast<long long>(tile) * kTile;
  const int Tt = static_cast<int>(min(static_cast<long long>(kTile), stream_len(p, s) - n0));
  const int nch = p.H / kBlk;
  const float* xrow0 = p.out + (static_cast<long long>(s) * p.n + n0) * p.H;
  const unsigned char* img_l = p.slot_img + static_cast<size_t>(l) * nch * 2 * kBlkBytes;
  bool ok = true;
  // The EMA field over the tile from zero [P3 §2.1 channel 2], per column:
  // A = sum over tokens r of (1-g) g^(Tt-1-r) x_r, so that the field after
  // the tile is g^Tt F + A; out_kernel's segments start from these.  The
  // last tile of an output segment also keeps its last kHalo x rows, the
  // ring window of the next segment's first tokens.
  __shared__ float s_fw[kTile];
  __shared__ __align__(16) float s_fpart[2][kBlk];  // read and written as float4
  if (tid < kTile) s_fw[tid] = tid < Tt ? (1.0f - p.ema_gamma) * powf(p.ema_gamma, static_cast<float>(Tt - 1 - tid)) : 0.f;
  float* fagg = reinterpret_cast<float*>(p.ws + p.ws_fagg) +
                (static_cast<long long>(s) * p.tiles_per_stream + tile) * p.H;
  const bool seg_end = (tile + 1) % p.tps_out == 0 && (tile + 1) * static_cast<long long>(kTile) < stream_len(p, s);
  float* halo = reinterpret_cast<float*>(p.ws + p.ws_halo) +
                (static_cast<long long>(s) * p.nseg_out + (tile + 1) / p.tps_out - 1) * kHalo * p.H;

  // Thread tid handles 4 columns c4 .. c4+3 of rows r_m (m = 0..3) of every
  // chunk.  The mapping makes a warp's split stores cover whole 128-byte
  // lines of the core-matrix layout (row r & 7 in lane bits 0-2, column bit
  // 2 in lane bit 3).
  const int c4 = ((tid >> 4) & 7) * 8 + ((tid >> 3) & 1) * 4;
  auto row_of = [&](int m) { return (2 * m + (tid >> 7)) * 8 + (tid & 7); };
  // x chunk c (columns 64c ..) into registers, rows past the tile zero.
  auto load_x = [&](int c, float4 (&v)[4]) {
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const int r = row_of(m);
      v[m] = r < Tt ? __ldcg(reinterpret_cast<const float4*>(xrow0 + static_cast<long long>(r) * p.H + c * kBlk + c4))
                    : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  };
  auto issue_img = [&](int c) {  // one thread; stage c % 3
    const int st = c % 3;
    mbar_arrive_expect_tx(bar_img + st, 2u * kBlkBytes);
    bulk_g2s(smb + PoolPlan::img + st * 2 * kBlkBytes, img_l + static_cast<size_t>(c) * 2 * kBlkBytes,
             2u * kBlkBytes, bar_img + st);
  };
  if (tid == 0) {
    issue_img(0);
    if (nch > 1) issue_img(1);
  }
  float4 nxt[4];
  load_x(0, nxt);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t idesc = umma_idesc_bf16(kBlk, kSlots, false);

  float sq[4] = {0.f, 0.f, 0.f, 0.f};  // |x|^2 of rows r_m over this thread's columns
  float s_fpart_keep[4];                // this half's field aggregate of the current chunk
  for (int c = 0; c < nch; ++c) {
    float4 cur[4];
#pragma unroll
    for (int m = 0; m < 4; ++m) cur[m] = nxt[m];
    if (c + 1 < nch) load_x(c + 1, nxt);  // in flight during this chunk
    const int st = c & 1;
    // The split blocks of stage st were read by the MMAs of chunk c-2.
    if (c >= 2 && !mbar_wait_bounded(bar_mma + st, static_cast<unsigned>(((c - 2) >> 1) & 1), kMbarPollLimit, p.err))
      ok = false;
    unsigned char* xhi = smb + PoolPlan::xsp + st * 2 * kBlkBytes;
    unsigned char* xlo = xhi + kBlkBytes;
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      const float4 v = cur[m];
      sq[m] = fmaf(v.x, v.x, fmaf(v.y, v.y, fmaf(v.z, v.z, fmaf(v.w, v.w, sq[m]))));
      __nv_bfloat16 hh[4], ll[4];
      split_bf16(v.x, hh[0], ll[0]);
      split_bf16(v.y, hh[1], ll[1]);
      split_bf16(v.z, hh[2], ll[2]);
      split_bf16(v.w, hh[3], ll[3]);
      const int off = blk_off(row_of(m), c4);
      *reinterpret_cast<uint2*>(xhi + off) = *reinterpret_cast<const uint2*>(hh);
      *reinterpret_cast<uint2*>(xlo + off) = *reinterpret_cast<const uint2*>(ll);
    }
    {  // field aggregate of the chunk's columns; halo rows of a segment end
      float fa[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const float wgt = s_fw[row_of(m)];
        fa[0] = fmaf(wgt, cur[m].x, fa[0]);
        fa[1] = fmaf(wgt, cur[m].y, fa[1]);
        fa[2] = fmaf(wgt, cur[m].z, fa[2]);
        fa[3] = fmaf(wgt, cur[m].w, fa[3]);
        if (seg_end && row_of(m) >= kTile - kHalo)
          *reinterpret_cast<float4*>(halo + static_cast<long long>(row_of(m) - (kTile - kHalo)) * p.H + c * kBlk + c4) = cur[m];
      }
#pragma unroll
      for (int e = 0; e < 4; ++e)  // the 8 lanes of this warp that share the columns
        for (int off = 1; off < 8; off <<= 1) fa[e] += __shfl_xor_sync(0xffffffffu, fa[e], off);
      if ((tid & 7) == 0 && (tid >> 7) == 1)
        *reinterpret_cast<float4*>(&s_fpart[c & 1][c4]) = make_float4(fa[0], fa[1], fa[2], fa[3]);
      s_fpart_keep[0] = fa[0];
      s_fpart_keep[1] = fa[1];
      s_fpart_keep[2] = fa[2];
      s_fpart_keep[3] = fa[3];
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();  // split blocks of chunk c written
    if ((tid & 7) == 0 && (tid >> 7) == 0) {  // the other half of the rows is in s_fpart
      const float4 o = *reinterpret_cast<const float4*>(&s_fpart[c & 1][c4]);
      *reinterpret_cast<float4*>(fagg + c * kBlk + c4) =
          make_float4(s_fpart_keep[0] + o.x, s_fpart_keep[1] + o.y, s_fpart_keep[2] + o.z, s_fpart_keep[3] + o.w);
    }
    if (tid == 0) {
      const int si = c % 3;
      if (!mbar_wait_bounded(bar_img + si, static_cast<unsigned>((c / 3) & 1), kMbarPollLimit, p.err)) ok = false;
      tc_fence_after();
      const unsigned char* shi = smb + PoolPlan::img + si * 2 * kBlkBytes;
      const unsigned char* slo = shi + kBlkBytes;
#pragma unroll
      for (int k = 0; k < kBlk / 16; ++k) {
        const uint64_t ah = umma_desc(xhi + k * 2048, 1024, 128), al = umma_desc(xlo + k * 2048, 1024, 128);
        const uint64_t bh = umma_desc(shi + k * 2048, 1024, 128), bl = umma_desc(slo + k * 2048, 1024, 128);
        umma_bf16(tmem, ah, bh, idesc, c > 0 || k > 0);
        umma_bf16(tmem, ah, bl, idesc, true);
        umma_bf16(tmem, al, bh, idesc, true);
      }
      umma_commit(bar_mma + st);
      if (c + 2 < nch) {
        // stage (c+2) % 3 held chunk c-1's slot blocks: wait for its MMAs
        // (committed one chunk ago), then reload it
        if (c >= 1 && !mbar_wait_bounded(bar_mma + ((c - 1) & 1), static_cast<unsigned>(((c - 1) >> 1) & 1),
                                         kMbarPollLimit, p.err))
          ok = false;
        issue_img(c + 2);
      }
    }
  }
  // |x|^2 per row: the 16 threads sharing a row add their partials in order.
#pragma unroll
  for (int m = 0; m < 4; ++m) sqp[((tid >> 3) & 15) * kTile + row_of(m)] = sq[m];
  __syncthreads();
  if (tid < kTile) {
    float v = 0.f;
#pragma unroll
    for (int q = 0; q < 16; ++q) v += sqp[q * kTile + tid];
    ssq[tid] = v;
  }
  // Test hook: a bounded wait on a barrier that nothing completes.
  if (tid == 0 && static_cast<long long>(tile) * p.n_streams + s == p.withhold_tile) {
    mbar_arrive_expect_tx(bar_probe, 16u);
    mbar_wait_bounded(bar_probe, 0, p.spin_limit, p.err);
  }
  {  // wait for the last MMAs (both stages' final commits)
    const int last = nch - 1;
    if (!mbar_wait_bounded(bar_mma + (last & 1), static_cast<unsigned>((last >> 1) & 1), kMbarPollLimit, p.err))
      ok = false;
    if (nch > 1 && !mbar_wait_bounded(bar_mma + ((last - 1) & 1),
                                      static_cast<unsigned>(((last - 1) >> 1) & 1), kMbarPollLimit, p.err))
      ok = false;
  }
  tc_fence_after();
  {  // accumulator row r (token) sits in lane (r%16) + 32*(r/16) for M = 64
    const int sp = warp & 3, colh = (warp >> 2) * 32;
    float v[32];
    tmem_ld32(tmem + (static_cast<uint32_t>(32 * sp) << 16) + colh, v);
    if (lane < 16) {
      float* dst = sc + (16 * sp + lane) * kScStride + colh;
#pragma unroll
      for (int j = 0; j < 32; ++j) dst[j] = v[j];
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }

  // softmax(cos/T) per token [P3 §2.1 channel 3]; weights split into bf16
  // hi/lo blocks in the MMA operand layout (in shared memory, where the x
  // split blocks were), then copied to the workspace.  Rows past the tile
  // get zero weights.
  const float* nrm = p.slot_norm + static_cast<size_t>(l) * kSlots;
  const float n0v = nrm[lane], n1v = nrm[lane + 32];
  unsigned char* wsm = smb + PoolPlan::xsp;
  for (int r = warp; r < kTile; r += NW) {
    float w0 = 0.f, w1 = 0.f;
    if (r < Tt) {
      const float nx = fmaxf(sqrtf(ssq[r]), kNormFloor);
      const float c0 = sc[r * kScStride + lane] / (nx * n0v) * p.inv_temp;
      const float c1 = sc[r * kScStride + lane + 32] / (nx * n1v) * p.inv_temp;
      const float mx = warp_max_redux(fmaxf(c0, c1));
      const float e0 = expf(c0 - mx), e1 = expf(c1 - mx);
      const float inv = 1.f / warp_sum(e0 + e1);
      w0 = e0 * inv;
      w1 = e1 * inv;
    }
    __nv_bfloat16 h0, l0, h1, l1;
    split_bf16(w0, h0, l0);
    split_bf16(w1, h1, l1);
    const int o0 = blk_off(r, lane), o1 = blk_off(r, lane + 32);
    *reinterpret_cast<__nv_bfloat16*>(wsm + o0) = h0;
    *reinterpret_cast<__nv_bfloat16*>(wsm + kBlkBytes + o0) = l0;
    *reinterpret_cast<__nv_bfloat16*>(wsm + o1) = h1;
    *reinterpret_cast<__nv_bfloat16*>(wsm + kBlkBytes + o1) = l1;
  }
  __syncthreads();
  uint4* wblk = reinterpret_cast<uint4*>(
      p.ws + p.ws_w + (static_cast<long long>(s) * p.tiles_per_stream + tile) * 2 * kBlkBytes);
  if (ok)
    for (int i = tid; i < 2 * kBlkBytes / 16; i += NT) wblk[i] = reinterpret_cast<const uint4*>(wsm)[i];
}

// ======================================================================
// 3. semantic mix, ring, field, fusion, output and state
// ======================================================================

struct OutPlan {
  static constexpr int bars = 0;                          // 5 mbarriers
  static constexpr int tmem = 64;
  static constexpr int img = 128;                         // [hi, lo] slot block of the columns
  static constexpr int wb = img + 2 * kBlkBytes;          // [2][hi, lo] weight blocks
  // [2][15 + 64][64] fp32: x of the 15 positions before the tile, then the tile
  static constexpr int xt = wb + 2 * 2 * kBlkBytes;
  static constexpr int sem = xt + 2 * (kHalo + kTile) * kBlk * 4;  // [64][65] sem
  static constexpr int segc = sem + kTile * kScStride * 4;  // [kSeg][64] field segment aggregates
  static constexpr int fcar = segc + kSeg * kBlk * 4;     // [64] field at the tile start
  static constexpr int total = fcar + kBlk * 4;
};

template <typename Tin>
__global__ void __launch_bounds__(NT, 2) out_kernel(const PrefillParams p) {
  const int ncb = p.H / kBlk;
  const int cb = static_cast<int>(blockIdx.x) % ncb;   // 64-column block
  const int seg = static_cast<int>(blockIdx.x) / ncb;  // segment of tiles
  const int s = blockIdx.y;                            // call-relative stream
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  extern __shared__ __align__(16) unsigned char smb[];
  uint64_t* bar_img = reinterpret_cast<uint64_t*>(smb + OutPlan::bars);
  uint64_t* bar_w = bar_img + 1;    // [2] weight blocks landed
  uint64_t* bar_mma = bar_img + 3;  // sem MMAs done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smb + OutPlan::tmem);
  float* semc = reinterpret_cast<float*>(smb + OutPlan::sem);
  float* segc = reinterpret_cast<float*>(smb + OutPlan::segc);
  float* fcar = reinterpret_cast<float*>(smb + OutPlan::fcar);
  __shared__ int s_ok;
  __shared__ long long s_pos;
  __shared__ float s_gseg[kSeg];

  pdl_trigger();
  pdl_wait();  // weights from pool_kernel (and, before it, x from near_kernel)
  unsigned char* blk = stream_block(p, s);
  if (tid == 0) {
    s_ok = header_matches(p);
    // the state's position is rewritten by this kernel: read the copy
    s_pos = reinterpret_cast<const long long*>(p.ws + p.ws_pos)[s];
    for (int b = 0; b < 4; ++b) mbar_init(bar_img + b, 1);
    mbar_fence_init();
  }
  __syncthreads();
  const long long ns = stream_len(p, s);  // tokens of this stream in the call
  const int tiles = static_cast<int>((ns + kTile - 1) / kTile);
  // this CTA's tiles: segment seg of the stream's tiles
  const int i_begin = seg * p.tps_out, i_end = min(tiles, i_begin + p.tps_out);
  if (!s_ok || i_begin >= i_end) return;  // an empty ragged stream keeps its state
  if (warp == 0) tmem_alloc(tmem_slot, kTmemCols);
  const long long pos0 = s_pos;
  const int l = p.l0 + s / p.B;
  const int col0 = cb * kBlk;
  const long long in_row0 = static_cast<long long>(s) * p.n;
  float* field = reinterpret_cast<float*>(blk + p.so.field);
  float* ring_sum = reinterpret_cast<float*>(blk + p.so.ring_sum);
  float* ring = reinterpret_cast<float*>(blk + p.so.ring);
  // the stream's pool weights (workspace pitch: the call's tiles per stream)
  const unsigned char* wall = p.ws + p.ws_w + static_cast<long long>(s) * p.tiles_per_stream * 2 * kBlkBytes;
  const float ge = p.ema_gamma;
  const float a_l = p.alpha_layer[l];

  auto tile_rows = [&](int i) -> int {
    return static_cast<int>(min(static_cast<long long>(kTile), ns - static_cast<long long>(i) * kTile));
  };
  constexpr int XR = kHalo + kTile;  // rows of an x stage
  auto xstage = [&](int st) -> float* { return reinterpret_cast<float*>(smb + OutPlan::xt) + st * XR * kBlk; };
  auto issue_x = [&](int i, int st) {
    float* xt = xstage(st) + kHalo * kBlk;
    const int Tt = tile_rows(i);
    const float* src = p.out + (in_row0 + static_cast<long long>(i) * kTile) * p.H + col0;
    for (int c = tid; c < Tt * (kBlk / 4); c += NT) {
      const int r = c / (kBlk / 4), c4 = (c % (kBlk / 4)) * 4;
      cp_async16(xt + r * kBlk + c4, src + static_cast<long long>(r) * p.H + c4);
    }
    cp_async_commit();
  };
  auto issue_w = [&](int i, int st) {  // one thread
    mbar_arrive_expect_tx(bar_w + st, 2u * kBlkBytes);
    bulk_g2s(smb + OutPlan::wb + st * 2 * kBlkBytes, wall + static_cast<long long>(i) * 2 * kBlkBytes,
             2u * kBlkBytes, bar_w + st);
  };
  if (tid == 0) {
    mbar_arrive_expect_tx(bar_img, 2u * kBlkBytes);
    bulk_g2s(smb + OutPlan::img,
             p.slot_img + (static_cast<size_t>(l) * (p.H / kBlk) + cb) * 2 * kBlkBytes, 2u * kBlkBytes,
             bar_img);
    issue_w(i_begin, 0);
  }
  issue_x(i_begin, 0);
  if (i_begin == 0) {
    // x of the 15 positions before the call (state ring; zero before
    // position 0) and the field carried in, for this block's columns.
    for (int idx = tid; idx < kHalo * kBlk; idx += NT) {
      const int q = idx / kBlk, c = idx % kBlk;
      const long long t = pos0 - kHalo + q;
      xstage(0)[idx] = t >= 0 ? ring[static_cast<size_t>(t % kRing) * p.H + col0 + c] : 0.f;
    }
    if (tid < kBlk) fcar[tid] = field[col0 + tid];
  } else {
    // a later segment: the last x rows of the previous segment, kept by
    // pool_kernel, and the field folded over the tiles before it (all full:
    // field after tile i = g^64 field + A_i)
    const float* halo = reinterpret_cast<const float*>(p.ws + p.ws_halo) +
                        (static_cast<long long>(s) * p.nseg_out + seg - 1) * kHalo * p.H + col0;
    for (int idx = tid; idx < kHalo * kBlk; idx += NT) {
      const int q = idx / kBlk, c = idx % kBlk;
      xstage(0)[idx] = halo[static_cast<long long>(q) * p.H + c];
    }
    if (tid < kBlk) {
      const float g64 = powf(ge, static_cast<float>(kTile));
      const float* agg = reinterpret_cast<const float*>(p.ws + p.ws_fagg) +
                         static_cast<long long>(s) * p.tiles_per_stream * p.H + col0 + tid;
      float f = field[col0 + tid];
      constexpr int kAhead = 8;  // aggregates in flight
      for (int i8 = 0; i8 < i_begin; i8 += kAhead) {
        float av[kAhead];
#pragma unroll
        for (int u = 0; u < kAhead; ++u) av[u] = i8 + u < i_begin ? agg[static_cast<long long>(i8 + u) * p.H] : 0.f;
#pragma unroll
        for (int u = 0; u < kAhead; ++u)
          if (i8 + u < i_begin) f = fmaf(g64, f, av[u]);
      }
      fcar[tid] = f;
    }
  }
  if (tid < kSeg) s_gseg[tid] = powf(ge, static_cast<float>(kSegLen));
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t idesc = umma_idesc_bf16(kTile, kBlk, true);
  bool ok = true;
  if (!mbar_wait_bounded(bar_img, 0, kMbarPollLimit, p.err)) ok = false;

  const int cc = tid % kBlk, sg = tid / kBlk;  // column, token segment
  for (int i = i_begin; i < i_end; ++i) {
    const int st = (i - i_begin) & 1;
    const int Tt = tile_rows(i);
    const long long t0 = pos0 + static_cast<long long>(i) * kTile;
    if (i + 1 < i_end) {
      issue_x(i + 1, st ^ 1);  // stage st^1 was released at the end of tile i-1
      if (tid == 0) issue_w(i + 1, st ^ 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    // sem[T x 64] = w[T x 64 slots] . slot block [64 slots x 64 columns]
    if (tid == 0) {
      if (!mbar_wait_bounded(bar_w + st, static_cast<unsigned>(((i - i_begin) >> 1) & 1), kMbarPollLimit, p.err)) ok = false;
      tc_fence_after();
      const unsigned char* whi = smb + OutPlan::wb + st * 2 * kBlkBytes;
      const unsigned char* wlo = whi + kBlkBytes;
      const unsigned char* shi = smb + OutPlan::img;
      const unsigned char* slo = shi + kBlkBytes;
#pragma unroll
      for (int k = 0; k < kSlots / 16; ++k) {
        const uint64_t ah = umma_desc(whi + k * 2048, 1024, 128), al = umma_desc(wlo + k * 2048, 1024, 128);
        const uint64_t bh = umma_desc(shi + k * 256, 128, 1024), bl = umma_desc(slo + k * 256, 128, 1024);
        umma_bf16(tmem, ah, bh, idesc, k > 0);
        umma_bf16(tmem, ah, bl, idesc, true);
        umma_bf16(tmem, al, bh, idesc, true);
      }
      umma_commit(bar_mma);
    }
    __syncthreads();  // x tile i visible to all threads
    // Thread (column cc, segment sg) owns tokens r_lo .. r_lo+15 of its
    // column.  Its x values for positions t0+r_lo-15 .. t0+r_lo+15 (stage
    // rows r_lo .. r_lo+30; rows past the tile hold stale values that no
    // result uses) go to registers in one batch.
    const float* xb = xstage(st);
    const int r_lo = sg * kSegLen;
    float xv[kSegLen + kHalo];
#pragma unroll
    for (int u = 0; u < kSegLen + kHalo; ++u) xv[u] = xb[(r_lo + u) * kBlk + cc];
    // field: this segment's aggregate from zero [P3 §2.1 channel 2]
    {
      float a = 0.f;
#pragma unroll
      for (int u = 0; u < kSegLen; ++u) {
        const float an = ewma(ge, a, xv[kHalo + u]);
        a = (r_lo + u < Tt) ? an : a;
      }
      segc[sg * kBlk + cc] = a;
    }
    if (!mbar_wait_bounded(bar_mma, static_cast<unsigned>((i - i_begin) & 1), kMbarPollLimit, p.err)) ok = false;
    tc_fence_after();
    {  // accumulator row r (token) sits in lane (r%16) + 32*(r/16) for M = 64
      const int sp = warp & 3, colh = (warp >> 2) * 32;
      float v[32];
      tmem_ld32(tmem + (static_cast<uint32_t>(32 * sp) << 16) + colh, v);
      if (lane < 16) {
        float* dst = semc + (16 * sp + lane) * kScStride + colh;
#pragma unroll
        for (int j = 0; j < 32; ++j) dst[j] = v[j];
      }
    }
    tc_fence_before();
    __syncthreads();
    float f = fcar[cc];
    for (int s2 = 0; s2 < sg; ++s2) f = fmaf(s_gseg[s2], f, segc[s2 * kBlk + cc]);
    float sv[kSegLen];
#pragma unroll
    for (int u = 0; u < kSegLen; ++u) sv[u] = semc[(r_lo + u) * kScStride + cc];
    // ring: sum of the 16 positions ending at token r [P3 §2.4: mean over all
    // 16 slots], sliding; fusion, clip and scale [P3 §2.2]
    float rs = 0.f;
#pragma unroll
    for (int u = 0; u < kRing; ++u) rs += xv[u];
    const long long orow = (in_row0 + (t0 - pos0) + r_lo) * p.H + col0 + cc;  // result element of token r_lo
#pragma unroll
    for (int u = 0; u < kSegLen; ++u) {
      if (u > 0) rs += xv[kHalo + u] - xv[u - 1];
      const float x = xv[kHalo + u];
      const bool live = r_lo + u < Tt;
      const float fn = ewma(ge, f, x);
      f = live ? fn : f;
      float uu = rs * (1.0f / kRing) + 0.5f * f + 0.5f * sv[u];
      uu = fminf(fmaxf(uu, -p.clip_eps), p.clip_eps);
      if (live && ok) store_result(p.out_mode, p.res, orow + static_cast<long long>(u) * p.H, a_l, uu, x);
    }
    const bool seg_last = r_lo < Tt && r_lo + kSegLen >= Tt;  // this segment holds the tile's last token
    if (i == tiles - 1 && ok) {  // the stream's last tile (in the last segment)
      const int gi = col0 + cc;
      if (seg_last) field[gi] = f;
      if (sg == 0) {
        // ring slots of the last 16 positions that belong to this call, and
        // the exact sum over all 16 (position q is stage row q - t0 + 15)
        const long long t_end = t0 + Tt - 1;
        float tot = 0.f;
        for (int r = 0; r < kRing; ++r) {
          const long long q = t_end - (kRing - 1) + r;
          if (q < 0) continue;
          const float v = xb[static_cast<int>(q - t0 + kHalo) * kBlk + cc];
          if (q >= pos0) ring[static_cast<size_t>(q % kRing) * p.H + gi] = v;
          tot += v;
        }
        ring_sum[gi] = tot;
      }
    }
    __syncthreads();  // segc and fcar are read above
    if (seg_last) fcar[cc] = f;
    if (i + 1 < i_end)  // the tile's last 15 x rows lead the next stage (Tt = 64 here)
      for (int idx = tid; idx < kHalo * kBlk; idx += NT) xstage(st ^ 1)[idx] = xb[kTile * kBlk + idx];
    __syncthreads();  // the x stage, halo rows and carries are ready for the next tile
  }

  // One CTA per stream (the last segment's): window, S and position [P1 §2.2].
  if (cb == 0 && i_end == tiles && ok) {
    unsigned char* b2 = blk;
    Tin* win_k = reinterpret_cast<Tin*>(b2 + p.so.win_k);
    Tin* win_v = reinterpret_cast<Tin*>(b2 + p.so.win_v);
    float* far = reinterpret_cast<float*>(b2 + p.so.far);
    const int D = p.H / p.nq;
    const float* sfin = reinterpret_cast<const float*>(p.ws + p.ws_sfin) + static_cast<long long>(s) * p.nkv * D;
    for (int idx = tid; idx < p.nkv * D; idx += NT) far[idx] = sfin[idx];
    const long long t_end = pos0 + ns - 1;
    const long long w0 = max(pos0, t_end - p.K + 1);
    const Tin* kin = static_cast<const Tin*>(p.k) + in_row0 * p.nkv * D;
    const Tin* vin = static_cast<const Tin*>(p.v) + in_row0 * p.nkv * D;
    const long long row = static_cast<long long>(p.nkv) * D;
    const long long cnt = (t_end - w0 + 1) * row;
    for (long long idx = tid; idx < cnt; idx += NT) {
      const long long j = w0 + idx / row, e = idx % row;
      win_k[(j % p.K) * row + e] = kin[(j - pos0) * row + e];
      win_v[(j % p.K) * row + e] = vin[(j - pos0) * row + e];
    }
    if (tid == 0) *reinterpret_cast<long long*>(b2 + p.so.pos) = pos0 + ns;
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------- host side

template <typename K>
cudaError_t set_smem(K kernel, int optin) {
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, kernel);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             optin - static_cast<int>(fa.sharedSizeBytes));
  return e;
}

template <typename K>
cudaError_t launch_pdl(K kernel, dim3 grid, int smem, cudaStream_t s, const PrefillParams& p) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(NT, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, p);
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link
// against the driver library).
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

// q as (D, n_q, rows) and k, v as (D, n_kv, rows) bf16 tensors, rows = every
// token of every stream of the call; boxes of 8 x 1 x T.
cudaError_t encode_near_maps(const PrefillParams& p, int D, NearMaps* m) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
  if (!enc) return cudaErrorNotSupported;
  const cuuint64_t rows = static_cast<cuuint64_t>(p.n_streams) * static_cast<cuuint64_t>(p.n);
  if (rows > 0x7fffffffULL) return cudaErrorInvalidValue;  // 32-bit coordinates
  const cuuint32_t estr[3] = {1, 1, 1};
  auto one = [&](CUtensorMap* map, const void* base, int heads, int box_rows) -> bool {
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(heads), rows};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(heads) * D * 2};
    const cuuint32_t box[3] = {8, 1, static_cast<cuuint32_t>(box_rows)};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
  };
  if (!one(&m->q, p.q, p.nq, kTile) || !one(&m->k, p.k, p.nkv, kNS) || !one(&m->v, p.v, p.nkv, kNS))
    return cudaErrorInvalidValue;
  return cudaSuccess;
}

template <typename Tin, int D>
cudaError_t launch_t(const PrefillParams& p, cudaStream_t s) {
  const unsigned ns = static_cast<unsigned>(p.n_streams);
  const int ne = p.nkv * D;
  const dim3 g0(static_cast<unsigned>(p.tiles_per_stream), ns, 1);
  const dim3 gc(static_cast<unsigned>((ne + NT - 1) / NT), ns, 1);
  const dim3 g1(static_cast<unsigned>(p.nq * p.n_seg), ns, 1);
  const dim3 g2(static_cast<unsigned>(p.tiles_per_stream), ns, 1);
  const dim3 g3(static_cast<unsigned>((p.H / kBlk) * p.nseg_out), ns, 1);
  cudaError_t e = launch_pdl(far_agg_kernel<Tin, D>, g0, 4 * ne * 4, s, p);
  if (e == cudaSuccess) e = launch_pdl(far_carry_kernel, gc, 0, s, p);
  if (e != cudaSuccess) return e;
  if constexpr (sizeof(Tin) == 2) {
    if (p.near.tc) {
      NearMaps maps;
      e = encode_near_maps(p, D, &maps);
      if (e == cudaSuccess) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = p.near.fused ? dim3(static_cast<unsigned>(p.n_seg), ns, 1) : g1;
        cfg.blockDim = dim3(p.near.fused ? NTF : NT, 1, 1);
        cfg.dynamicSmemBytes = static_cast<size_t>(p.near.total);
        cfg.stream = s;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        e = p.near.fused ? cudaLaunchKernelEx(&cfg, fused_kernel<D>, p, maps)
                         : cudaLaunchKernelEx(&cfg, near_tc_kernel<D>, p, maps);
      }
    } else {
      e = launch_pdl(near_kernel<Tin, D>, g1, p.near.total, s, p);
    }
  } else {
    e = launch_pdl(near_kernel<Tin, D>, g1, p.near.total, s, p);
  }
  if (e == cudaSuccess && !p.near.fused) e = launch_pdl(pool_kernel, g2, p.pool_smem, s, p);
  if (e == cudaSuccess) e = launch_pdl(out_kernel<Tin>, g3, p.out_smem, s, p);
  return e;
}

}  // namespace

bool plan_near(int D, int esz, int K, size_t limit, bool tc, bool fused, NearPlan* out) {
  auto a16 = [](long long x) { return static_cast<int>((x + 15) & ~15LL); };
  NearPlan p;
  std::memset(&p, 0, sizeof(p));
  tc = tc && esz == 2 && K <= 16;
  p.tc = tc ? 1 : 0;
  if (tc && fused) {
    p.fused = 1;
    p.total = D == 64 ? FusedPlan<64>::total : FusedPlan<128>::total;
    if (static_cast<size_t>(p.total) > limit) return false;
    *out = p;
    return true;
  }
  p.row = D * esz + 16;
  const int xs = a16(4LL * kTile * (D + kXsPad));
  const int qb = tc ? kTile * D * 2 : a16(static_cast<long long>(kTile) * p.row);
  const int kvb = tc ? (D / 8) * kDStr : a16(static_cast<long long>(kTile + K) * p.row);
  const int fixed = tc ? 2 * (2 * kTile * kNS * 2) : xs;  // P and G blocks, or the x tile
  const int stage = qb + 2 * kvb;
  // Two stages where they keep two CTAs per SM, else one, else (CUDA cores)
  // keys and values from global memory (windows too wide to stage).
  const long long two_per_sm = static_cast<long long>(limit) / 2 - 1024;
  int stages = 0;
  if (2LL * stage + fixed <= two_per_sm) stages = 2;
  else if (static_cast<long long>(stage) + fixed <= two_per_sm) stages = 1;
  else if (2LL * stage + fixed <= static_cast<long long>(limit)) stages = 2;
  else if (static_cast<long long>(stage) + fixed <= static_cast<long long>(limit)) stages = 1;
  if (tc && stages == 0) return false;
  int off = 0;
  if (tc) {
    p.pa = off;
    off += 2 * kTile * kNS * 2;
    p.ga = off;
    off += 2 * kTile * kNS * 2;
  } else {
    p.xs = off;
    off += xs;
  }
  for (int st = 0; st < 2; ++st) {
    if (st < std::max(stages, 1)) {
      p.q[st] = off;
      off += qb;
      if (stages > 0) {
        p.k[st] = off;
        off += kvb;
        p.v[st] = off;
        off += kvb;
      }
    } else {
      p.q[st] = p.q[0];
      p.k[st] = p.k[0];
      p.v[st] = p.v[0];
    }
  }
  p.stages = stages;
  p.total = off + (tc ? 128 : 0);  // tensor cores: slack to align the base to 128 bytes
  if (static_cast<size_t>(p.total) > limit) return false;
  *out = p;
  return true;
}

int prefill_pool_smem() { return PoolPlan::total; }
int prefill_out_smem() { return OutPlan::total; }

cudaError_t prefill_prepare(int device) {
  int optin = 0;
  cudaError_t e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, device);
  if (e == cudaSuccess) e = set_smem(near_kernel<float, 64>, optin);
  if (e == cudaSuccess) e = set_smem(near_kernel<float, 128>, optin);
  if (e == cudaSuccess) e = set_smem(near_kernel<__nv_bfloat16, 64>, optin);
  if (e == cudaSuccess) e = set_smem(near_kernel<__nv_bfloat16, 128>, optin);
  if (e == cudaSuccess) e = set_smem(near_tc_kernel<64>, optin);
  if (e == cudaSuccess) e = set_smem(near_tc_kernel<128>, optin);
  if (e == cudaSuccess) e = set_smem(fused_kernel<64>, optin);
  if (e == cudaSuccess) e = set_smem(fused_kernel<128>, optin);
  if (e == cudaSuccess) e = set_smem(far_agg_kernel<float, 64>, optin);
  if (e == cudaSuccess) e = set_smem(far_agg_kernel<float, 128>, optin);
  if (e == cudaSuccess) e = set_smem(far_agg_kernel<__nv_bfloat16, 64>, optin);
  if (e == cudaSuccess) e = set_smem(far_agg_kernel<__nv_bfloat16, 128>, optin);
  if (e == cudaSuccess) e = set_smem(pool_kernel, optin);
  if (e == cudaSuccess) e = set_smem(out_kernel<float>, optin);
  if (e == cudaSuccess) e = set_smem(out_kernel<__nv_bfloat16>, optin);
  return e;
}

size_t prefill_smem_limit(int device) {
  int optin = 0;
  if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, device) != cudaSuccess)
    return 0;
  return static_cast<size_t>(optin) - 1024;  // headroom for the kernels' static shared memory
}

cudaError_t launch_prefill(const PrefillParams& p, int in_dtype, int head_dim, cudaStream_t s) {
  if (in_dtype == SFA_F32) return head_dim == 64 ? launch_t<float, 64>(p, s) : launch_t<float, 128>(p, s);
  return head_dim == 64 ? launch_t<__nv_bfloat16, 64>(p, s) : launch_t<__nv_bfloat16, 128>(p, s);
}

}  // namespace sfa
