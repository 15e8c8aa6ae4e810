// sfa_decode_tile.cu — SFA decode step for large batches, in two kernels
// chained by programmatic dependent launch; every state update in place.
//
// Sources (web pages):
//   [P1] "Signal Field Attention (SFA)：8KB代码实现4.16倍推理加速与248倍内存压缩"
//        §2.1 eqs. O_near, S_t, O; §2.2 O(k·d) window state.
//   [P3] "Dalin Soma SFA基于信号场注意力机制的神经网络推理加速框架"
//        §2.1 channels 1–3, §2.2 fusion, clip and alpha_layer, §2.4 ring mean.
//
// At a batch of hundreds a decode step streams about 150 KB per (layer,
// sequence) through HBM; what limits it is how many bytes each SM keeps in
// flight and how many SMs take part.  Neither kernel uses clusters, so every
// SM takes part, and each keeps its loads in flight ahead of the arithmetic.
//
// decode_near_kernel: near field [P1 §2.1 eq. O_near], far field [eq. S_t]
//   and x = O_near + alpha_far·S [eq. O].  A CTA serves a block of
//   sequences of one layer; its work items are (sequence, KV head), all the
//   KV head's query heads at once, so every window is read once.  Each warp
//   runs its own items with two header buffers (q rows, K_t, V_t, S) and two
//   window buffers (16 slots of keys and values), filled by bulk and tensor
//   copies counted in bytes on mbarriers: the next item's copies are in
//   flight while the warp computes.  An online softmax over the chunks and
//   P·V run on the CUDA cores.  x goes into `out`, which holds it until the
//   pool kernel overwrites it; the warp then writes K_t, V_t into window
//   slot t mod k and the new S (it alone read them).
// decode_pool_kernel: semantic pool [P3 §2.1 channel 3], ring, field,
//   fusion, clip and output [P3 §2.1, §2.2].  A CTA serves 16 sequences of
//   one layer over the whole hidden vector, in 64-column chunks: pass 1
//   feeds x through split bf16 blocks (hi*hi + hi*lo + lo*hi, about 16
//   significant bits) to the tcgen05 tensor cores against the pre-split slot
//   blocks, scores[16 x 64] accumulating in tensor memory, and sums |x|^2;
//   softmax(cos/T) gives the weights; pass 2 forms sem = w . slot chunk by
//   chunk on the tensor cores and runs the epilogue, with x and the state
//   rows of the next chunks already loading.  The MMAs use M = 64 with the
//   rows past the 16 sequences zero.
//
// Every wait is bounded; a wait that runs out latches SFA_ERR_DEVICE_TIMEOUT
// and the kernel still finishes.
#include <cooperative_groups.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstring>

#include "sfa_common.cuh"
#include "sfa_umma.cuh"

namespace cg = cooperative_groups;

namespace sfa {
namespace {

constexpr int NTN = 256;                // near-field kernel threads
constexpr int NWN = NTN / 32;
constexpr int HB = kDecodeTileHeads;    // query heads per KV head served
constexpr int KCB = kDecodeTileChunk;   // window slots per chunk
constexpr int kPbFloats = HB * KCB + 2 * HB;  // per warp: P, corrections, denominators
constexpr int kNearRowsMax = 32;        // most sequences per near-field CTA (chosen per launch)
static_assert(HB <= 8 && KCB == 16, "near-field lane mapping: 2 x 16 lanes, 4 heads each");

// Tensor maps of one call: the state's window rings (keys, values) as
// (head dim, KV head, slot, stream) views with boxes of one KV head x kcb
// slots; for bf16 inputs also q as (head dim, query head, input row) with
// boxes of one KV head's query heads, both in 64-dim halves with 128-byte
// swizzling.
struct WinMaps {
  CUtensorMap k, v, q;
};

__host__ __device__ inline int a128(long long x) { return static_cast<int>((x + 127) & ~127LL); }

__device__ __forceinline__ unsigned char* aligned128(unsigned char* p) {
  return reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(p) + 127) & ~static_cast<uintptr_t>(127));
}

// Near-field CTA shared memory: [barriers: 4 per warp][P buffers][per warp:
// header 0, header 1, chunk 0, chunk 1].
constexpr int kNearBarBytes = 128 * ((NWN * 4 * 8 + 127) / 128);
constexpr int kNearPbBytes = 128 * ((NWN * kPbFloats * 4 + 127) / 128);

template <typename Tin, int D>
__global__ void __launch_bounds__(NTN, 1)
decode_near_kernel(const __grid_constant__ DecodeParams p, const __grid_constant__ WinMaps maps) {
  constexpr int ESZ = static_cast<int>(sizeof(Tin));
  constexpr int VE = Load16<Tin>::N;  // elements per 16-byte load
  constexpr int NC16 = D / VE;        // 16-byte chunks of one head row
  constexpr int DPL = D / 32;         // head dims per lane in P·V
  static_assert((NC16 & (NC16 - 1)) == 0, "row chunks must be a power of two");
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const TilePlan& pl = p.tp;
  const int K = p.K, G = p.G, nkv = p.nkv;
  const int rows = p.tp.near_rows;  // sequences of this CTA's block
  const int blocks_per_layer = (p.n_seq + rows - 1) / rows;
  const int li = static_cast<int>(blockIdx.x) / blocks_per_layer;
  const int rb = static_cast<int>(blockIdx.x) % blocks_per_layer;
  const int l = p.l0 + li;
  const int kcb = pl.kcb;
  const int nck = (K + kcb - 1) / kcb;

  extern __shared__ __align__(128) unsigned char smb_raw[];
  unsigned char* sm = aligned128(smb_raw);  // the plan leaves 128 bytes of slack
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm) + warp * 4;  // hdr full [2], chunk full [2]
  float* pbw = reinterpret_cast<float*>(sm + kNearBarBytes) + warp * kPbFloats;
  float* pP = pbw;                // [HB][KCB] softmax numerators of the chunk
  float* pCorr = pbw + HB * KCB;  // [HB] rescale of the running sums
  float* pDen = pCorr + HB;       // [HB] final denominators
  unsigned char* wbase = sm + kNearBarBytes + kNearPbBytes + warp * pl.warp_bytes;
  auto hdr = [&](int i) { return wbase + i * pl.hdr_bytes; };                        // headers 0, 1
  auto chk = [&](int i) { return wbase + 2 * pl.hdr_bytes + i * pl.chunk_bytes; };   // chunks 0, 1
  __shared__ long long s_st[kNearRowsMax], s_pos[kNearRowsMax];

  if (lane == 0) {
    for (int i = 0; i < 4; ++i) mbar_init(bars + i, 1);
    mbar_fence_init();
  }
  pdl_trigger();
  pdl_wait();  // state and inputs may be written by the previous kernel
  if (tid < rows) {  // the block's sequences: stream index and position
    const int bi = rb * rows + tid;
    long long st = -1, ps = 0;
    if (bi < p.n_seq) {
      const int b = p.seq_ids ? __ldcg(p.seq_ids + bi) : bi;
      if (b >= 0 && b < p.B) {
        st = static_cast<long long>(l) * p.B + b;
        ps = __ldcg(reinterpret_cast<const long long*>(p.state + kHeaderBytes + st * p.so.stride + p.so.pos));
      } else {
        latch_error(p.err, SFA_ERR_INVALID_ARG);
      }
    }
    s_st[tid] = st;
    s_pos[tid] = ps;
  }
  __syncthreads();
  {
    const uint4 h0v = __ldcg(reinterpret_cast<const uint4*>(p.state));
    const uint4 h1v = __ldcg(reinterpret_cast<const uint4*>(p.state + 16));
    StateHeader hd;
    reinterpret_cast<uint4*>(&hd)[0] = h0v;
    reinterpret_cast<uint4*>(&hd)[1] = h1v;
    if (!(hd.magic == kMagic && hd.cfg_hash == p.cfg_hash && hd.batch == p.B && hd.n_layers == p.L)) {
      if (tid == 0 && blockIdx.x == 0) latch_error(p.err, SFA_ERR_STATE_MISMATCH);
      return;  // the same answer in every CTA; no copy was issued
    }
  }

  // Items of this warp: it = warp, warp + NWN, ... of (row, KV head) pairs.
  const int n_items = rows * nkv;
  const long long in_row0 = static_cast<long long>(li) * p.n_seq + static_cast<long long>(rb) * rows;
  auto item_row = [&](int it) { return it / nkv; };
  // Copies of one unit (item `it`, window chunk `piece`) into chunk buffer
  // `b`; the header (into header buffer `hb`) with piece 0.  Lane 0 only.
  // For an absent sequence the barriers get a plain arrival instead, so
  // every buffer's phases advance once per unit either way.
  auto issue = [&](int it, int piece, int b, int hb) {
    const int r = item_row(it), g = it - r * nkv;
    const long long st = s_st[r];
    if (st < 0) {
      if (piece == 0) mbar_arrive(bars + hb);
      mbar_arrive(bars + 2 + b);
      return;
    }
    fence_proxy_async_smem();  // this warp's reads of the buffers came first
    if (piece == 0) {
      uint64_t* hf = bars + hb;
      const long long io = in_row0 + r;
      mbar_arrive_expect_tx(hf, static_cast<unsigned>((G + 2) * D * ESZ + 4 * D));
      bulk_g2s(hdr(hb) + pl.hq, static_cast<const Tin*>(p.q) + (io * p.nq + static_cast<long long>(g) * G) * D,
               static_cast<unsigned>(G * D * ESZ), hf);
      bulk_g2s(hdr(hb) + pl.hkt, static_cast<const Tin*>(p.k) + (io * nkv + g) * D, D * ESZ, hf);
      bulk_g2s(hdr(hb) + pl.hvt, static_cast<const Tin*>(p.v) + (io * nkv + g) * D, D * ESZ, hf);
      bulk_g2s(hdr(hb) + pl.hs, p.state + kHeaderBytes + st * p.so.stride + p.so.far + static_cast<long long>(g) * D * 4,
               D * 4, hf);
    }
    uint64_t* cf = bars + 2 + b;
    mbar_arrive_expect_tx(cf, static_cast<unsigned>(2 * kcb * D * ESZ));
    tma_load_4d(chk(b), &maps.k, 0, g, piece * kcb, static_cast<int>(st), cf);
    tma_load_4d(chk(b) + kcb * D * ESZ, &maps.v, 0, g, piece * kcb, static_cast<int>(st), cf);
  };

  // QK: lane (j, half) scores chunk slot j against heads half, half+2,
  // half+4, half+6; each lane starts its walk along the head row at 16-byte
  // chunk j, so the lanes of a half hit distinct banks.  P·V: lane owns head
  // dims lane*DPL .. +DPL of every head.
  const int j = lane & 15, half = lane >> 4, d0 = lane * DPL;
  bool ok = true;
  int unit = 0;  // units (item, chunk) of this warp so far: chunk buffer unit & 1
  int k_item = 0;
  if (lane == 0 && warp < n_items) issue(warp, 0, 0, 0);
  for (int it = warp; it < n_items; it += NWN, ++k_item) {
    const int r = item_row(it), g = it - r * nkv;
    const long long st = s_st[r];
    const long long t = s_pos[r];
    const int es = static_cast<int>(t % K);  // slot of token t: holds the evicted key t-k
    const bool full_win = t >= K - 1;        // every slot holds a position >= 0
    const int hb = k_item & 1;
    const Tin* qh = reinterpret_cast<const Tin*>(hdr(hb) + pl.hq);
    const Tin* ktr = reinterpret_cast<const Tin*>(hdr(hb) + pl.hkt);
    const Tin* vtr = reinterpret_cast<const Tin*>(hdr(hb) + pl.hvt);
    const float* s_old = reinterpret_cast<const float*>(hdr(hb) + pl.hs);
    float mrun[4], drun[4], o[HB][DPL], kev[DPL];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      mrun[u] = -INFINITY;
      drun[u] = 0.f;
    }
#pragma unroll
    for (int hh = 0; hh < HB; ++hh)
#pragma unroll
      for (int e = 0; e < DPL; ++e) o[hh][e] = 0.f;
#pragma unroll
    for (int e = 0; e < DPL; ++e) kev[e] = 0.f;
    if (!mbar_wait_bounded(bars + hb, static_cast<unsigned>((k_item >> 1) & 1), kMbarPollLimit, p.err)) ok = false;
    for (int piece = 0; piece < nck; ++piece) {
      const int b = unit & 1;
      // the next unit's copies go out before this one is computed
      if (lane == 0) {
        if (piece + 1 < nck) issue(it, piece + 1, b ^ 1, hb);
        else if (it + NWN < n_items) issue(it + NWN, 0, b ^ 1, hb ^ 1);
      }
      if (!mbar_wait_bounded(bars + 2 + b, static_cast<unsigned>((unit >> 1) & 1), kMbarPollLimit, p.err))
        ok = false;
      ++unit;
      if (st < 0) continue;
      const Tin* kc = reinterpret_cast<const Tin*>(chk(b));
      const Tin* vc = kc + kcb * D;
      // scores of slot s = piece*kcb + j; slot es holds token t itself
      const int s = piece * kcb + j;
      const bool valid = j < kcb && s < K && (full_win || s <= t);
      float sc[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) sc[u] = -INFINITY;
      if (valid) {
        const Tin* krow = (s == es) ? ktr : kc + j * D;
        float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
        for (int cc = 0; cc < NC16; ++cc) {
          const int ch = (cc + j) & (NC16 - 1);
          float kv[VE];
          Load16<Tin>::run(krow + ch * VE, kv);
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            if (half + 2 * u < G) {
              float qv[VE];
              Load16<Tin>::run(qh + (half + 2 * u) * D + ch * VE, qv);
#pragma unroll
              for (int e = 0; e < VE; ++e) acc[u] = fmaf(qv[e], kv[e], acc[u]);
            }
          }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) sc[u] = acc[u] * p.score_scale;
      }
      // online softmax over the chunk's slots, per head (16 lanes)
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int hh = half + 2 * u;
        float cm = sc[u];
#pragma unroll
        for (int off = 8; off > 0; off >>= 1) cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, off));
        const float mn = fmaxf(mrun[u], cm);
        const bool any = mn != -INFINITY;
        const float corr = any ? expf(mrun[u] - mn) : 1.f;
        const float pj = (sc[u] != -INFINITY) ? expf(sc[u] - mn) : 0.f;
        float ps = pj;
#pragma unroll
        for (int off = 8; off > 0; off >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
        drun[u] = fmaf(drun[u], corr, ps);
        mrun[u] = mn;
        if (hh < G) {
          pP[hh * KCB + j] = pj;
          if (j == 0) pCorr[hh] = corr;
        }
      }
      __syncwarp();
      // P·V over the chunk's valid slots (uniform over the warp)
#pragma unroll
      for (int hh = 0; hh < HB; ++hh) {
        if (hh < G) {
          const float cr = pCorr[hh];
#pragma unroll
          for (int e = 0; e < DPL; ++e) o[hh][e] *= cr;
        }
      }
      const int rows = min(kcb, K - piece * kcb);
      for (int jj = 0; jj < rows; ++jj) {
        const int s2 = piece * kcb + jj;
        if (!(full_win || s2 <= t)) continue;
        const Tin* vrow = (s2 == es) ? vtr : vc + jj * D;
        float vv[DPL];
        VecLoad<Tin, DPL>::run(vrow + d0, vv);
#pragma unroll
        for (int hh = 0; hh < HB; ++hh) {
          if (hh < G) {
            const float pv = pP[hh * KCB + jj];
#pragma unroll
            for (int e = 0; e < DPL; ++e) o[hh][e] = fmaf(pv, vv[e], o[hh][e]);
          }
        }
      }
      // the key that token t evicts (the old content of slot es)
      if (piece == es / kcb) VecLoad<Tin, DPL>::run(kc + (es - piece * kcb) * D + d0, kev);
      __syncwarp();
    }
    if (st < 0) continue;
    // x = O_near + alpha_far * S_t into out; then the window slot and S
    if (j == 0) {
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (half + 2 * u < G) pDen[half + 2 * u] = drun[u];
    }
    __syncwarp();
    const long long io = in_row0 + r;
    float sn[DPL];
#pragma unroll
    for (int e = 0; e < DPL; ++e) sn[e] = (t >= K) ? ewma(p.gamma_far, s_old[d0 + e], kev[e]) : s_old[d0 + e];
    float* xrow = p.out + io * p.H + static_cast<long long>(g) * G * D + d0;
#pragma unroll
    for (int hh = 0; hh < HB; ++hh) {
      if (hh < G) {
        const float inv = 1.f / pDen[hh];
        float v[DPL];
#pragma unroll
        for (int e = 0; e < DPL; ++e) v[e] = fmaf(p.alpha_far, sn[e], o[hh][e] * inv);
        if constexpr (DPL == 4) {
          *reinterpret_cast<float4*>(xrow + hh * D) = make_float4(v[0], v[1], v[2], v[3]);
        } else {
          *reinterpret_cast<float2*>(xrow + hh * D) = make_float2(v[0], v[1]);
        }
      }
    }
    if (ok) {
      unsigned char* blk = p.state + kHeaderBytes + st * p.so.stride;
      float* far = reinterpret_cast<float*>(blk + p.so.far) + g * D + d0;
#pragma unroll
      for (int e = 0; e < DPL; ++e) far[e] = sn[e];
      const size_t wo = (static_cast<size_t>(es) * nkv + g) * D + d0;
      Tin* win_k = reinterpret_cast<Tin*>(blk + p.so.win_k) + wo;
      Tin* win_v = reinterpret_cast<Tin*>(blk + p.so.win_v) + wo;
#pragma unroll
      for (int e = 0; e < DPL; ++e) {
        win_k[e] = ktr[d0 + e];
        win_v[e] = vtr[d0 + e];
      }
    }
    __syncwarp();  // pDen and the header are reused by the next items
  }
}

// ---------------------------------------------------- near field, bf16 MMAs

// Warp-level bf16 matrix ops: ldmatrix (four 8 x 8 b16 matrices, optionally
// transposed) and mma.sync m16n8k16 with fp32 accumulation.
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo_col, float hi_col) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo_col, hi_col);  // .x = first (lower) column
  return *reinterpret_cast<const uint32_t*>(&v);
}

// Shared-memory layout of the MMA near field, per warp (bytes): two headers
// then two window chunks.  A header holds the q rows of the item's query
// heads as (head dim / 64) swizzled 1 KB blocks of 8 rows x 128 bytes, then
// K_t, V_t (plain) and S (fp32).  A chunk holds keys then values, each as
// (head dim / 64) swizzled blocks of 16 slots x 128 bytes.  Tensor copies
// with 128-byte swizzling put the 16-byte group j of row r at group
// j ^ (r % 8); every block starts on a 1 KB boundary.
template <int D>
struct MmaNear {
  static constexpr int NH = D / 64;              // 64-dim halves of a head row
  static constexpr int qblk = 1024;              // 8 rows x 128 B
  static constexpr int hq = 0;
  static constexpr int hkt = NH * qblk;
  static constexpr int hvt = hkt + D * 2;
  static constexpr int hs = hvt + D * 2;
  static constexpr int hdr = ((hs + 4 * D + 1023) / 1024) * 1024;
  static constexpr int kblk = KCB * 128;         // 16 rows x 128 B
  static constexpr int chunk = 2 * NH * kblk;    // keys, then values
  static constexpr int warp = 2 * hdr + 2 * chunk;
};

template <int D>
__global__ void __launch_bounds__(NTN, 1)
decode_near_mma_kernel(const __grid_constant__ DecodeParams p, const __grid_constant__ WinMaps maps) {
  using L = MmaNear<D>;
  constexpr int NT16 = D / 8;  // n-tiles of 8 head dims
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int K = p.K, G = p.G, nkv = p.nkv;
  const int rows = p.tp.near_rows;  // sequences of this CTA's block
  const int blocks_per_layer = (p.n_seq + rows - 1) / rows;
  const int li = static_cast<int>(blockIdx.x) / blocks_per_layer;
  const int rb = static_cast<int>(blockIdx.x) % blocks_per_layer;
  const int l = p.l0 + li;
  const int kcb = p.tp.kcb;
  const int nck = (K + kcb - 1) / kcb;

  extern __shared__ __align__(128) unsigned char smb_mma[];
  // 1 KB aligned base (the plan leaves 1 KB of slack) for the swizzled blocks
  unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smb_mma) + 1023) &
                                                       ~static_cast<uintptr_t>(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm) + warp * 4;  // hdr full [2], chunk full [2]
  unsigned char* wbase = sm + 1024 + warp * L::warp;
  auto hdr = [&](int i) { return wbase + i * L::hdr; };
  auto chk = [&](int i) { return wbase + 2 * L::hdr + i * L::chunk; };
  __shared__ long long s_st[kNearRowsMax], s_pos[kNearRowsMax];

  if (lane == 0) {
    for (int i = 0; i < 4; ++i) mbar_init(bars + i, 1);
    mbar_fence_init();
  }
  if (kcb < KCB) {  // slots past kcb are never copied: keep them finite (zero)
    for (int b = 0; b < 2; ++b)
      for (int i = lane; i < 2 * L::NH * (KCB - kcb) * 8; i += 32) {
        const int blk = i / ((KCB - kcb) * 8), rem = i % ((KCB - kcb) * 8);
        reinterpret_cast<uint4*>(chk(b) + blk * L::kblk + kcb * 128)[rem] = make_uint4(0u, 0u, 0u, 0u);
      }
  }
  pdl_trigger();
  pdl_wait();  // state and inputs may be written by the previous kernel
  if (tid < rows) {
    const int bi = rb * rows + tid;
    long long st = -1, ps = 0;
    if (bi < p.n_seq) {
      const int b = p.seq_ids ? __ldcg(p.seq_ids + bi) : bi;
      if (b >= 0 && b < p.B) {
        st = static_cast<long long>(l) * p.B + b;
        ps = __ldcg(reinterpret_cast<const long long*>(p.state + kHeaderBytes + st * p.so.stride + p.so.pos));
      } else {
        latch_error(p.err, SFA_ERR_INVALID_ARG);
      }
    }
    s_st[tid] = st;
    s_pos[tid] = ps;
  }
  __syncthreads();
  {
    const uint4 h0v = __ldcg(reinterpret_cast<const uint4*>(p.state));
    const uint4 h1v = __ldcg(reinterpret_cast<const uint4*>(p.state + 16));
    StateHeader hd;
    reinterpret_cast<uint4*>(&hd)[0] = h0v;
    reinterpret_cast<uint4*>(&hd)[1] = h1v;
    if (!(hd.magic == kMagic && hd.cfg_hash == p.cfg_hash && hd.batch == p.B && hd.n_layers == p.L)) {
      if (tid == 0 && blockIdx.x == 0) latch_error(p.err, SFA_ERR_STATE_MISMATCH);
      return;
    }
  }

  const int n_items = rows * nkv;
  const long long in_row0 = static_cast<long long>(li) * p.n_seq + static_cast<long long>(rb) * rows;
  // Copies of one unit into chunk buffer b (header buffer hb with piece 0);
  // lane 0.  Absent sequences: plain arrivals, so phases stay in step.
  auto issue = [&](int it, int piece, int b, int hb) {
    const int r = it / nkv, g = it - r * nkv;
    const long long st = s_st[r];
    if (st < 0) {
      if (piece == 0) mbar_arrive(bars + hb);
      mbar_arrive(bars + 2 + b);
      return;
    }
    fence_proxy_async_smem();  // this warp's accesses of the buffers came first
    if (piece == 0) {
      uint64_t* hf = bars + hb;
      const long long io = in_row0 + r;
      unsigned char* h = hdr(hb);
      mbar_arrive_expect_tx(hf, static_cast<unsigned>((G + 2) * D * 2 + 4 * D));
#pragma unroll
      for (int hh = 0; hh < L::NH; ++hh)
        tma_load_3d(h + L::hq + hh * L::qblk, &maps.q, 64 * hh, g * G, static_cast<int>(io), hf);
      bulk_g2s(h + L::hkt, static_cast<const __nv_bfloat16*>(p.k) + (io * nkv + g) * D, D * 2, hf);
      bulk_g2s(h + L::hvt, static_cast<const __nv_bfloat16*>(p.v) + (io * nkv + g) * D, D * 2, hf);
      bulk_g2s(h + L::hs, p.state + kHeaderBytes + st * p.so.stride + p.so.far + static_cast<long long>(g) * D * 4,
               D * 4, hf);
    }
    uint64_t* cf = bars + 2 + b;
    unsigned char* c = chk(b);
    mbar_arrive_expect_tx(cf, static_cast<unsigned>(2 * kcb * D * 2));
#pragma unroll
    for (int hh = 0; hh < L::NH; ++hh) {
      tma_load_4d(c + hh * L::kblk, &maps.k, 64 * hh, g, piece * kcb, static_cast<int>(st), cf);
      tma_load_4d(c + (L::NH + hh) * L::kblk, &maps.v, 64 * hh, g, piece * kcb, static_cast<int>(st), cf);
    }
  };

  const int g8 = lane >> 2, tig = lane & 3;  // MMA fragment row / column pair
  const int mi = lane >> 3, rr = lane & 7;   // ldmatrix: matrix and row this lane addresses
  bool ok = true;
  int unit = 0;
  int k_item = 0;
  if (lane == 0 && warp < n_items) issue(warp, 0, 0, 0);
  for (int it = warp; it < n_items; it += NWN, ++k_item) {
    const int r = it / nkv, g = it - r * nkv;
    const long long st = s_st[r];
    const long long t = s_pos[r];
    const int es = static_cast<int>(t % K);  // slot of token t: holds the evicted key t-k
    const bool full_win = t >= K - 1;
    const int hb = k_item & 1;
    unsigned char* h = hdr(hb);
    const uint32_t qb = smem_u32(h + L::hq);
    const __nv_bfloat16* ktr = reinterpret_cast<const __nv_bfloat16*>(h + L::hkt);
    const __nv_bfloat16* vtr = reinterpret_cast<const __nv_bfloat16*>(h + L::hvt);
    const float* s_old = reinterpret_cast<const float*>(h + L::hs);
    float o[NT16][4], kev[NT16][2];
#pragma unroll
    for (int n = 0; n < NT16; ++n) {
      o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
      kev[n][0] = kev[n][1] = 0.f;
    }
    float m_run = -INFINITY, l_run = 0.f;  // row g8 of the item (query head g8)
    if (!mbar_wait_bounded(bars + hb, static_cast<unsigned>((k_item >> 1) & 1), kMbarPollLimit, p.err)) ok = false;
    for (int piece = 0; piece < nck; ++piece) {
      const int b = unit & 1;
      if (lane == 0) {
        if (piece + 1 < nck) issue(it, piece + 1, b ^ 1, hb);
        else if (it + NWN < n_items) issue(it + NWN, 0, b ^ 1, hb ^ 1);
      }
      if (!mbar_wait_bounded(bars + 2 + b, static_cast<unsigned>((unit >> 1) & 1), kMbarPollLimit, p.err))
        ok = false;
      ++unit;
      if (st < 0) continue;
      unsigned char* c = chk(b);
      const uint32_t kb = smem_u32(c), vb = smem_u32(c + L::NH * L::kblk);
      const int base = piece * kcb;
      if (piece == es / kcb) {
        // slot es holds the key token t evicts: keep it for S, then put
        // token t's own key and value in its place
        const int er = es - base;
#pragma unroll
        for (int n = 0; n < NT16; ++n) {
          const __nv_bfloat162 e2 = *reinterpret_cast<const __nv_bfloat162*>(
              c + (n >> 3) * L::kblk + er * 128 + (((n & 7) ^ (er & 7)) << 4) + 4 * tig);
          const float2 f = __bfloat1622float2(e2);
          kev[n][0] = f.x;
          kev[n][1] = f.y;
        }
        __syncwarp();
        if (lane < 2 * NT16) {  // 16-byte groups of K_t (lanes < NT16) and V_t
          const int grp = lane % NT16;
          const bool is_v = lane >= NT16;
          const uint4 src = *reinterpret_cast<const uint4*>((is_v ? vtr : ktr) + 8 * grp);
          *reinterpret_cast<uint4*>(c + ((is_v ? L::NH : 0) + (grp >> 3)) * L::kblk + er * 128 +
                                    (((grp & 7) ^ (er & 7)) << 4)) = src;
        }
        __syncwarp();
      }
      // S[16 heads x 16 slots] = q . K^T; heads >= G read head 0 (discarded)
      float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        uint32_t a[4], bk[4];
        int qrow = rr + 8 * (mi & 1);
        if (qrow >= G) qrow = 0;
        const int qg = 2 * ks + (mi >> 1);
        ldsm_x4(qb + (qg >> 3) * L::qblk + qrow * 128 + (((qg & 7) ^ (qrow & 7)) << 4), a);
        const int krow = rr + 8 * (mi >> 1);
        const int kg = 2 * ks + (mi & 1);
        ldsm_x4(kb + (kg >> 3) * L::kblk + krow * 128 + (((kg & 7) ^ (krow & 7)) << 4), bk);
        mma16816(s0, a, bk[0], bk[1]);
        mma16816(s1, a, bk[2], bk[3]);
      }
      // online softmax for row g8 over the chunk's valid slots
      float v[4] = {s0[0], s0[1], s1[0], s1[1]};
      float cm = -INFINITY;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int kk = (e >> 1) * 8 + 2 * tig + (e & 1);
        const int s = base + kk;
        const bool valid = kk < kcb && s < K && (full_win || s <= t);
        v[e] = valid ? v[e] * p.score_scale : -INFINITY;
        cm = fmaxf(cm, v[e]);
      }
      cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, 1));
      cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, 2));
      const float mn = fmaxf(m_run, cm);
      const float corr = mn == -INFINITY ? 1.f : expf(m_run - mn);
      float pr[4], ps = 0.f;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        pr[e] = v[e] == -INFINITY ? 0.f : expf(v[e] - mn);
        ps += pr[e];
      }
      ps += __shfl_xor_sync(0xffffffffu, ps, 1);
      ps += __shfl_xor_sync(0xffffffffu, ps, 2);
      l_run = fmaf(l_run, corr, ps);
      m_run = mn;
      if (piece > 0) {
#pragma unroll
        for (int n = 0; n < NT16; ++n) {
          o[n][0] *= corr;
          o[n][1] *= corr;
        }
      }
      // P as split bf16 A operands (rows 8..15 zero): P = P_hi + P_lo
      uint32_t ah[4], al[4];
      {
        float hi[4], lo[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          hi[e] = __bfloat162float(__float2bfloat16_rn(pr[e]));
          lo[e] = pr[e] - hi[e];
        }
        ah[0] = pack_bf16(hi[0], hi[1]);
        ah[1] = 0u;
        ah[2] = pack_bf16(hi[2], hi[3]);
        ah[3] = 0u;
        al[0] = pack_bf16(lo[0], lo[1]);
        al[1] = 0u;
        al[2] = pack_bf16(lo[2], lo[3]);
        al[3] = 0u;
      }
      // O[16 x D] += P . V over the chunk's 16 slots
#pragma unroll
      for (int n2 = 0; n2 < NT16 / 2; ++n2) {
        uint32_t bv[4];
        const int vrow = rr + 8 * (mi & 1);
        const int vg = 2 * n2 + (mi >> 1);
        ldsm_x4_t(vb + (vg >> 3) * L::kblk + vrow * 128 + (((vg & 7) ^ (vrow & 7)) << 4), bv);
        mma16816(o[2 * n2], ah, bv[0], bv[1]);
        mma16816(o[2 * n2], al, bv[0], bv[1]);
        mma16816(o[2 * n2 + 1], ah, bv[2], bv[3]);
        mma16816(o[2 * n2 + 1], al, bv[2], bv[3]);
      }
      __syncwarp();
    }
    if (st < 0) continue;
    // x = O_near + alpha_far * S_t for the item's heads; then S and slot es
    const long long io = in_row0 + r;
    const float inv = 1.f / l_run;
    float* far = reinterpret_cast<float*>(p.state + kHeaderBytes + st * p.so.stride + p.so.far) + g * D;
    float* xrow = p.out + io * p.H + (static_cast<long long>(g) * G + g8) * D;
#pragma unroll
    for (int n = 0; n < NT16; ++n) {
      const int d = 8 * n + 2 * tig;
      float sn0 = s_old[d], sn1 = s_old[d + 1];
      if (t >= K) {
        sn0 = ewma(p.gamma_far, sn0, kev[n][0]);
        sn1 = ewma(p.gamma_far, sn1, kev[n][1]);
      }
      if (g8 < G)
        *reinterpret_cast<float2*>(xrow + d) =
            make_float2(fmaf(p.alpha_far, sn0, o[n][0] * inv), fmaf(p.alpha_far, sn1, o[n][1] * inv));
      if (g8 == 0 && ok) *reinterpret_cast<float2*>(far + d) = make_float2(sn0, sn1);
    }
    if (ok && lane < 2 * NT16) {
      const int grp = lane % NT16;
      const bool is_v = lane >= NT16;
      const size_t wo = (static_cast<size_t>(es) * nkv + g) * D + 8 * grp;
      unsigned char* blk = p.state + kHeaderBytes + st * p.so.stride;
      __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(blk + (is_v ? p.so.win_v : p.so.win_k)) + wo;
      *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>((is_v ? vtr : ktr) + 8 * grp);
    }
    __syncwarp();  // the header is reused two items later
  }
}

// ---------------------------------------------------------------- pool kernel

// The split x^T and w^T blocks ([16 x 64] bf16, core-matrix layout) keep
// their 8-column groups kGrp16 = 256 + 16 bytes apart: the 16 lanes that
// write one row then spread over all 32 banks (256 apart they share four).
// As a K-major MMA operand the next K group is kGrp16 bytes on.
constexpr int kGrp16 = 272;
constexpr int kBlk16Pad = 8 * kGrp16;
__device__ __forceinline__ int pad16_off(int row, int col) {
  return (col >> 3) * kGrp16 + (row >> 3) * kCoreBytes + (row & 7) * 16 + (col & 7) * 2;
}

constexpr int NTC = 256;                // pool kernel: compute threads (8 warps)
constexpr int NWC = NTC / 32;
constexpr int NTP = NTC + 32;           // plus the MMA warp
constexpr int TR = 16;                  // sequences per CTA pair: the N = 16 of the MMAs
constexpr int kPair = 2;                // CTAs of a cluster: halves of the hidden columns
constexpr int kSlotStages = 4;
constexpr int kABufs = 4;               // split x^T blocks
constexpr int kSemBufs = 4;             // sem^T accumulators and their staging
constexpr int kScStride = kSlots + 1;   // 64 scores + |x|^2 per row
constexpr int kSemStride = kBlk + 4;
constexpr int kTmemCols = 128;          // scores^T (16) + four 16-column sem^T buffers
constexpr int kTmemSem = 32;
static_assert(TR * 16 == NTC, "pool kernel: 16 threads per row, 4 columns each");

// Pool CTA shared memory (byte offsets).
struct PoolTilePlan {
  static constexpr int bars = 0;                                  // mbarriers, tmem address
  static constexpr int sl = 1024;                                 // [4][hi, lo] slot blocks
  static constexpr int xt = sl + kSlotStages * 2 * kBlkBytes;     // [4][hi, lo] x^T blocks [16 x 64]
  static constexpr int wt = xt + kABufs * 2 * kBlk16Pad;        // [hi, lo] w^T block [16 x 64]
  static constexpr int sem = wt + 2 * kBlk16Pad;                // [4][16][68] sem chunks
  static constexpr int sc = sem + kSemBufs * TR * kSemStride * 4; // [16][65] own partial scores, |x|^2
  static constexpr int scp = sc + TR * kScStride * 4;             // [16][65] the peer CTA's partial
  static constexpr int total = scp + TR * kScStride * 4;
};
// barrier slots (arrival counts in brackets)
constexpr int kPbSlFull = 0;                           // [4] slot block landed (1 + bytes)
constexpr int kPbSlEmpty = kPbSlFull + kSlotStages;    // [4] MMAs done with a slot block (commit)
constexpr int kPbAFull = kPbSlEmpty + kSlotStages;     // [4] x^T block written (8 warps)
constexpr int kPbAEmpty = kPbAFull + kABufs;           // [4] MMAs done with an x^T block (commit)
constexpr int kPbScores = kPbAEmpty + kABufs;          // all score MMAs done (commit)
constexpr int kPbWFull = kPbScores + 1;                // w^T block written (8 warps)
constexpr int kPbSemFull = kPbWFull + 1;               // [4] sem accumulator ready (commit)
constexpr int kPbSemEmpty = kPbSemFull + kSemBufs;     // [4] sem accumulator read (4 warps)
constexpr int kPbStFull = kPbSemEmpty + kSemBufs;      // [4] sem chunk staged (4 warps)
constexpr int kPbStEmpty = kPbStFull + kSemBufs;       // [4] staged sem chunk used (8 warps)
constexpr int kPbCount = kPbStEmpty + kSemBufs;
static_assert(kPbCount * 8 + 4 <= PoolTilePlan::sl, "barriers fit");

// A cluster of two CTAs serves 16 sequences of one layer; CTA `rank` owns
// the hidden columns of chunks [c0, c0 + nloc).  The 16 sequences are the
// N = 16 of transposed MMAs: scores^T[64 slots x 16] += slot_c . x_c^T and
// sem^T[64 columns x 16] = slot_c^T . w^T, split bf16 operands (hi*hi +
// hi*lo + lo*hi), fp32 accumulators in tensor memory.  The two CTAs add
// their partial scores and |x|^2 through distributed shared memory and both
// form the same softmax weights.  Warp 8 (one lane) loads the slot blocks
// and issues every MMA; warps 0-7 split x (pass 1) and run the epilogue
// with x and the state rows two chunks ahead in registers (pass 2); warps
// 0-3, which hold the accumulator lanes, stage each sem chunk for the
// others.  mbarriers carry every hand-off.
__global__ void __cluster_dims__(kPair, 1, 1) __launch_bounds__(NTP, 2)
decode_pool_kernel(const __grid_constant__ DecodeParams p) {
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = static_cast<int>(cluster.block_rank());
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int tiles_per_layer = (p.n_seq + TR - 1) / TR;
  const int pair = static_cast<int>(blockIdx.x) / kPair;
  const int li = pair / tiles_per_layer;
  const int tb = pair % tiles_per_layer;
  const int l = p.l0 + li;
  const int nch = p.H / kBlk;
  const int half = (nch + 1) / 2;
  const int c0 = rank == 0 ? 0 : half;
  const int nloc = rank == 0 ? half : nch - half;  // chunks of this CTA
  extern __shared__ __align__(128) unsigned char smb_pool[];
  unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smb_pool) + 127) &
                                                       ~static_cast<uintptr_t>(127));
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + PoolTilePlan::bars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kPbCount);
  unsigned char* slb = sm + PoolTilePlan::sl;
  unsigned char* xtb = sm + PoolTilePlan::xt;
  unsigned char* wtb = sm + PoolTilePlan::wt;
  float* semst = reinterpret_cast<float*>(sm + PoolTilePlan::sem);
  float* sc = reinterpret_cast<float*>(sm + PoolTilePlan::sc);
  float* scp = reinterpret_cast<float*>(sm + PoolTilePlan::scp);
  __shared__ long long s_st[TR], s_pos[TR];
  __shared__ int s_ok;

  const unsigned char* img_l = p.slot_img + static_cast<size_t>(l) * nch * 2 * kBlkBytes;
  // Slot block loads q = 0 .. 2*nloc-1 (pass 1, then pass 2): load q is
  // block c0 + q % nloc in stage q % 4.
  auto issue_slot = [&](int q) {  // the MMA lane
    const int st = q % kSlotStages;
    mbar_arrive_expect_tx(bars + kPbSlFull + st, 2u * kBlkBytes);
    bulk_g2s(slb + st * 2 * kBlkBytes, img_l + static_cast<size_t>(c0 + q % nloc) * 2 * kBlkBytes,
             2u * kBlkBytes, bars + kPbSlFull + st);
  };
  if (tid == 0) {
    for (int i = 0; i < kPbCount; ++i) {
      int count = 1;
      if ((i >= kPbAFull && i < kPbAFull + kABufs) || i == kPbWFull || (i >= kPbStEmpty && i < kPbStEmpty + kSemBufs))
        count = NWC;
      if ((i >= kPbSemEmpty && i < kPbSemEmpty + kSemBufs) || (i >= kPbStFull && i < kPbStFull + kSemBufs)) count = 4;
      mbar_init(bars + i, count);
    }
    mbar_fence_init();
  }
  if (warp == 0) tmem_alloc(tmem_slot, kTmemCols);  // at most two CTAs per SM: never waits
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // The peer writes into this CTA's shared memory only after every CTA of
  // the cluster has started: arrive now, wait before the exchange.
  cluster_arrive();
  if (warp == NWC && lane == 0) {
    // the slot blocks are constant since sfa_init: the first loads go out
    // before the wait for the previous kernel
    for (int q = 0; q < kSlotStages && q < 2 * nloc; ++q) issue_slot(q);
  }
  pdl_trigger();
  pdl_wait();  // x from the near-field kernel; the state

  if (tid == 0) {
    const uint4 h0v = __ldcg(reinterpret_cast<const uint4*>(p.state));
    const uint4 h1v = __ldcg(reinterpret_cast<const uint4*>(p.state + 16));
    StateHeader hd;
    reinterpret_cast<uint4*>(&hd)[0] = h0v;
    reinterpret_cast<uint4*>(&hd)[1] = h1v;
    s_ok = hd.magic == kMagic && hd.cfg_hash == p.cfg_hash && hd.batch == p.B && hd.n_layers == p.L;
  }
  if (tid < TR) {
    const int bi = tb * TR + tid;
    long long st = -1, ps = 0;
    if (bi < p.n_seq) {
      const int b = p.seq_ids ? __ldcg(p.seq_ids + bi) : bi;
      if (b >= 0 && b < p.B) {
        st = static_cast<long long>(l) * p.B + b;
        ps = __ldcg(reinterpret_cast<const long long*>(p.state + kHeaderBytes + st * p.so.stride + p.so.pos));
      }
    }
    s_st[tid] = st;
    s_pos[tid] = ps;
  }
  __syncthreads();
  bool ok = s_ok != 0;  // a mismatch was latched by the near-field kernel
  const uint32_t idesc_s = umma_idesc_bf16_ab(kBlk, TR, false, false);  // slot (K-major) . x^T (K-major)
  const uint32_t idesc_c = umma_idesc_bf16_ab(kBlk, TR, true, false);   // slot^T (MN-major) . w^T

  if (warp == NWC) {
    // ---- MMA warp: slot loads and every MMA -------------------------------
    if (lane == 0) {
      // After the MMAs of load q: the stage of load q-1 (its MMAs committed
      // one chunk earlier) takes load q + 3.
      auto refill_slot = [&](int q) {
        if (q < 1 || q + kSlotStages - 1 >= 2 * nloc) return;
        const int st = (q - 1) % kSlotStages;
        if (!mbar_wait_bounded(bars + kPbSlEmpty + st, static_cast<unsigned>(((q - 1) / kSlotStages) & 1),
                               kMbarPollLimit, p.err))
          ok = false;
        issue_slot(q + kSlotStages - 1);
      };
      // pass 1: scores^T[64 slots x 16] += slot_c . x_c^T over this CTA's chunks
      for (int c = 0; c < nloc; ++c) {
        const int stg = c % kSlotStages, b = c % kABufs;
        if (!mbar_wait_bounded(bars + kPbSlFull + stg, static_cast<unsigned>((c / kSlotStages) & 1), kMbarPollLimit, p.err))
          ok = false;
        if (!mbar_wait_bounded(bars + kPbAFull + b, static_cast<unsigned>((c / kABufs) & 1), kMbarPollLimit, p.err))
          ok = false;
        tc_fence_after();
        const unsigned char* shi = slb + stg * 2 * kBlkBytes;
        const unsigned char* xhi = xtb + b * 2 * kBlk16Pad;
#pragma unroll
        for (int k = 0; k < kBlk / 16; ++k) {
          const uint64_t ah = umma_desc(shi + k * 2048, 1024, 128), al = umma_desc(shi + kBlkBytes + k * 2048, 1024, 128);
          const uint64_t bh = umma_desc(xhi + k * 2 * kGrp16, kGrp16, 128), bl = umma_desc(xhi + kBlk16Pad + k * 2 * kGrp16, kGrp16, 128);
          umma_bf16(tmem, ah, bh, idesc_s, c > 0 || k > 0);
          umma_bf16(tmem, ah, bl, idesc_s, true);
          umma_bf16(tmem, al, bh, idesc_s, true);
        }
        umma_commit(bars + kPbAEmpty + b);
        umma_commit(bars + kPbSlEmpty + stg);
        refill_slot(c);
      }
      umma_commit(bars + kPbScores);
    }
    __syncwarp();
    cluster_wait();    // phase 1: both CTAs started
    cluster_arrive();  // phase 2: the partials are exchanged
    cluster_wait();
    if (lane == 0) {
      auto refill_slot = [&](int q) {
        if (q < 1 || q + kSlotStages - 1 >= 2 * nloc) return;
        const int st = (q - 1) % kSlotStages;
        if (!mbar_wait_bounded(bars + kPbSlEmpty + st, static_cast<unsigned>(((q - 1) / kSlotStages) & 1),
                               kMbarPollLimit, p.err))
          ok = false;
        issue_slot(q + kSlotStages - 1);
      };
      // pass 2: sem^T chunk c [64 columns x 16] = slot_c^T . w^T
      if (!mbar_wait_bounded(bars + kPbWFull, 0, kMbarPollLimit, p.err)) ok = false;
      for (int c = 0; c < nloc; ++c) {
        const int q = nloc + c, stg = q % kSlotStages, b = c % kSemBufs;
        if (!mbar_wait_bounded(bars + kPbSlFull + stg, static_cast<unsigned>((q / kSlotStages) & 1), kMbarPollLimit, p.err))
          ok = false;
        if (c >= kSemBufs && !mbar_wait_bounded(bars + kPbSemEmpty + b, static_cast<unsigned>(((c / kSemBufs) - 1) & 1),
                                                kMbarPollLimit, p.err))
          ok = false;
        tc_fence_after();
        const uint32_t dst = tmem + kTmemSem + b * TR;
        const unsigned char* shi = slb + stg * 2 * kBlkBytes;
#pragma unroll
        for (int k = 0; k < kSlots / 16; ++k) {
          const uint64_t ah = umma_desc(shi + k * 256, 128, 1024), al = umma_desc(shi + kBlkBytes + k * 256, 128, 1024);
          const uint64_t bh = umma_desc(wtb + k * 2 * kGrp16, kGrp16, 128), bl = umma_desc(wtb + kBlk16Pad + k * 2 * kGrp16, kGrp16, 128);
          umma_bf16(dst, ah, bh, idesc_c, k > 0);
          umma_bf16(dst, ah, bl, idesc_c, true);
          umma_bf16(dst, al, bh, idesc_c, true);
        }
        umma_commit(bars + kPbSemFull + b);
        umma_commit(bars + kPbSlEmpty + stg);
        refill_slot(q);
      }
    }
    __syncwarp();
  } else {
    // ---- compute warps: thread tid owns row r = tid / 16, columns c4 .. c4+3
    const int r = tid >> 4, c4 = (tid & 15) * 4;
    const long long st = s_st[r];
    const long long io = static_cast<long long>(li) * p.n_seq + static_cast<long long>(tb) * TR + r;
    const bool live = st >= 0 && ok;
    const float* xrow = p.out + (live ? io : 0) * p.H + c0 * kBlk + c4;
    auto load_x = [&](int c) -> float4 {
      return (live && c < nloc) ? __ldcg(reinterpret_cast<const float4*>(xrow + c * kBlk))
                                : make_float4(0.f, 0.f, 0.f, 0.f);
    };
    // pass 1: x chunk c into x^T block c % 4 (split bf16), |x|^2
    float4 xn0 = load_x(0), xn1 = load_x(1);  // chunks c and c+1 in flight
    float sq = 0.f;
    for (int c = 0; c < nloc; ++c) {
      const int b = c % kABufs;
      const float4 v = xn0;
      xn0 = xn1;
      xn1 = load_x(c + 2);
      sq = fmaf(v.x, v.x, fmaf(v.y, v.y, fmaf(v.z, v.z, fmaf(v.w, v.w, sq))));
      if (c >= kABufs &&
          !mbar_wait_bounded(bars + kPbAEmpty + b, static_cast<unsigned>(((c / kABufs) - 1) & 1), kMbarPollLimit, p.err))
        ok = false;
      unsigned char* xhi = xtb + b * 2 * kBlk16Pad;
      __nv_bfloat16 hh[4], ll[4];
      split_bf16(v.x, hh[0], ll[0]);
      split_bf16(v.y, hh[1], ll[1]);
      split_bf16(v.z, hh[2], ll[2]);
      split_bf16(v.w, hh[3], ll[3]);
      const int off = pad16_off(r, c4);
      *reinterpret_cast<uint2*>(xhi + off) = *reinterpret_cast<const uint2*>(hh);
      *reinterpret_cast<uint2*>(xhi + kBlk16Pad + off) = *reinterpret_cast<const uint2*>(ll);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(bars + kPbAFull + b);
    }
#pragma unroll
    for (int off = 8; off > 0; off >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, off);
    // partial scores and |x|^2 of this CTA's columns, into its own and the
    // peer's shared memory
    float* peer_scp = cluster.map_shared_rank(scp, rank ^ 1);
    cluster_wait();  // phase 1: the peer has started
    if ((tid & 15) == 0) {
      sc[r * kScStride + kSlots] = sq;
      peer_scp[r * kScStride + kSlots] = sq;
    }
    if (warp < 4) {  // slot 16w + i sits in lane i of lane quarter w (M = 64)
      if (!mbar_wait_bounded(bars + kPbScores, 0, kMbarPollLimit, p.err)) ok = false;
      tc_fence_after();
      float v[16];
      if (nloc > 0) {
        tmem_ld16(tmem + (static_cast<uint32_t>(32 * warp) << 16), v);
      } else {
#pragma unroll
        for (int rr = 0; rr < TR; ++rr) v[rr] = 0.f;
      }
      if (lane < 16) {
#pragma unroll
        for (int rr = 0; rr < TR; ++rr) {
          sc[rr * kScStride + 16 * warp + lane] = v[rr];
          peer_scp[rr * kScStride + 16 * warp + lane] = v[rr];
        }
      }
    }
    __syncwarp();
    cluster_arrive();  // phase 2: both partials in place
    cluster_wait();
    // softmax(cos/T) per row [P3 §2.1 channel 3]; weights as split bf16 w^T
    {
      const float* nrm = p.slot_norm + static_cast<size_t>(l) * kSlots;
      const float n0 = nrm[lane], n1 = nrm[lane + 32];
      for (int rr = warp; rr < TR; rr += NWC) {
        const float* a = sc + rr * kScStride;
        const float* b = scp + rr * kScStride;
        const float nx = fmaxf(sqrtf(a[kSlots] + b[kSlots]), kNormFloor);
        const float c0v = (a[lane] + b[lane]) / (nx * n0) * p.inv_temp;
        const float c1v = (a[lane + 32] + b[lane + 32]) / (nx * n1) * p.inv_temp;
        const float mx = warp_max_redux(fmaxf(c0v, c1v));
        const float e0 = expf(c0v - mx), e1 = expf(c1v - mx);
        const float inv = 1.f / warp_sum(e0 + e1);
        __nv_bfloat16 h0, l0, h1, l1;
        split_bf16(e0 * inv, h0, l0);
        split_bf16(e1 * inv, h1, l1);
        const int o0 = pad16_off(rr, lane), o1 = pad16_off(rr, lane + 32);
        *reinterpret_cast<__nv_bfloat16*>(wtb + o0) = h0;
        *reinterpret_cast<__nv_bfloat16*>(wtb + kBlk16Pad + o0) = l0;
        *reinterpret_cast<__nv_bfloat16*>(wtb + o1) = h1;
        *reinterpret_cast<__nv_bfloat16*>(wtb + kBlk16Pad + o1) = l1;
      }
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(bars + kPbWFull);

    // pass 2: ring, field, fusion, clip, output [P3 §2.1 channels 1-2, §2.2]
    const int slot_r = static_cast<int>(s_pos[r] & (kRing - 1));
    unsigned char* blk = p.state + kHeaderBytes + (live ? st : 0) * p.so.stride;
    float* ring_r = reinterpret_cast<float*>(blk + p.so.ring) + static_cast<size_t>(slot_r) * p.H + c0 * kBlk + c4;
    float* rsum_r = reinterpret_cast<float*>(blk + p.so.ring_sum) + c0 * kBlk + c4;
    float* fld_r = reinterpret_cast<float*>(blk + p.so.field) + c0 * kBlk + c4;
    float* out_r = p.out + (live ? io : 0) * p.H + c0 * kBlk + c4;
    struct Row4 {
      float4 x, old, rs, fl;
    };
    auto load_row = [&](int c) -> Row4 {
      Row4 v;
      if (live && c < nloc) {
        v.x = __ldcg(reinterpret_cast<const float4*>(out_r + c * kBlk));
        v.old = __ldcg(reinterpret_cast<const float4*>(ring_r + c * kBlk));
        v.rs = __ldcg(reinterpret_cast<const float4*>(rsum_r + c * kBlk));
        v.fl = __ldcg(reinterpret_cast<const float4*>(fld_r + c * kBlk));
      } else {
        v.x = v.old = v.rs = v.fl = make_float4(0.f, 0.f, 0.f, 0.f);
      }
      return v;
    };
    Row4 rn0 = load_row(0), rn1 = load_row(1);  // chunks c and c+1 in flight
    const float a_l = p.alpha_layer[l];
    for (int c = 0; c < nloc; ++c) {
      const int b = c % kSemBufs;
      const unsigned ph = static_cast<unsigned>((c / kSemBufs) & 1);
      float* sstg = semst + b * TR * kSemStride;
      if (warp < 4) {
        // accumulator b (column 16w + i in lane i, rows along columns) ->
        // sem staging b, once the compute warps are done with it
        if (!mbar_wait_bounded(bars + kPbSemFull + b, ph, kMbarPollLimit, p.err)) ok = false;
        tc_fence_after();
        float v[16];
        tmem_ld16(tmem + (static_cast<uint32_t>(32 * warp) << 16) + kTmemSem + b * TR, v);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bars + kPbSemEmpty + b);
        if (c >= kSemBufs && !mbar_wait_bounded(bars + kPbStEmpty + b, static_cast<unsigned>(((c / kSemBufs) - 1) & 1),
                                                kMbarPollLimit, p.err))
          ok = false;
        if (lane < 16) {
#pragma unroll
          for (int rr = 0; rr < TR; ++rr) sstg[rr * kSemStride + 16 * warp + lane] = v[rr];
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(bars + kPbStFull + b);
      }
      const Row4 cur = rn0;
      rn0 = rn1;
      rn1 = load_row(c + 2);
      if (!mbar_wait_bounded(bars + kPbStFull + b, ph, kMbarPollLimit, p.err)) ok = false;
      const float4 sv = *reinterpret_cast<const float4*>(sstg + r * kSemStride + c4);
      __syncwarp();
      if (lane == 0) mbar_arrive(bars + kPbStEmpty + b);
      if (live && ok) {
        const float xa[4] = {cur.x.x, cur.x.y, cur.x.z, cur.x.w};
        const float roa[4] = {cur.old.x, cur.old.y, cur.old.z, cur.old.w};
        const float rsa[4] = {cur.rs.x, cur.rs.y, cur.rs.z, cur.rs.w};
        const float fla[4] = {cur.fl.x, cur.fl.y, cur.fl.z, cur.fl.w};
        const float sva[4] = {sv.x, sv.y, sv.z, sv.w};
        float rv[4], fv[4], ov[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          rv[e] = (rsa[e] - roa[e]) + xa[e];        // ring sum after storing x_t
          fv[e] = ewma(p.ema_gamma, fla[e], xa[e]);  // EMA field
          float uu = rv[e] * (1.0f / kRing) + 0.5f * fv[e] + 0.5f * sva[e];
          uu = fminf(fmaxf(uu, -p.clip_eps), p.clip_eps);
          ov[e] = fmaf(a_l, uu, xa[e]);
        }
        *reinterpret_cast<float4*>(ring_r + c * kBlk) = cur.x;
        *reinterpret_cast<float4*>(rsum_r + c * kBlk) = make_float4(rv[0], rv[1], rv[2], rv[3]);
        *reinterpret_cast<float4*>(fld_r + c * kBlk) = make_float4(fv[0], fv[1], fv[2], fv[3]);
        *reinterpret_cast<float4*>(out_r + c * kBlk) = make_float4(ov[0], ov[1], ov[2], ov[3]);
      }
    }
    if (rank == 0 && live && ok && (tid & 15) == 0)
      *reinterpret_cast<long long*>(p.state + kHeaderBytes + st * p.so.stride + p.so.pos) = s_pos[r] + 1;
  }

  // every tensor-core operation has completed (the last sem chunk was read)
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------- host side

template <typename K>
cudaError_t set_smem_t(K kernel, int optin) {
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, kernel);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             optin - static_cast<int>(fa.sharedSizeBytes));
  return e;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no link
// against the driver library).
PFN_cuTensorMapEncodeTiled_v12000 tile_map_encoder() {
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

// The window rings of every stream of the state as (head dim, KV head,
// slot, stream) tensors: boxes of head_dim x 1 x kcb x 1 (fp32 inputs), or
// of 64 x 1 x kcb x 1 with 128-byte swizzling (bf16 inputs, warp MMAs),
// which then also get q as a (head dim, query head, input row) tensor.
cudaError_t encode_win_maps(const DecodeParams& p, int D, int esz, WinMaps* m) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tile_map_encoder();
  if (!enc) return cudaErrorNotSupported;
  const bool mma = esz == 2;
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(p.nkv),
                              static_cast<cuuint64_t>(p.K),
                              static_cast<cuuint64_t>(p.L) * static_cast<cuuint64_t>(p.B)};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(D) * esz, static_cast<cuuint64_t>(p.nkv) * D * esz,
                                 static_cast<cuuint64_t>(p.so.stride)};
  const cuuint32_t box[4] = {static_cast<cuuint32_t>(mma ? 64 : D), 1, static_cast<cuuint32_t>(p.tp.kcb), 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUtensorMapDataType dt = esz == 4 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const CUtensorMapSwizzle sw = mma ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE;
  auto one = [&](CUtensorMap* map, long long off) -> bool {
    void* base = p.state + kHeaderBytes + off;
    return enc(map, dt, 4, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
  };
  if (!one(&m->k, p.so.win_k) || !one(&m->v, p.so.win_v)) return cudaErrorInvalidValue;
  std::memset(&m->q, 0, sizeof(m->q));
  if (mma) {
    const cuuint64_t qdims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(p.nq),
                                 static_cast<cuuint64_t>(p.Lc) * static_cast<cuuint64_t>(p.n_seq)};
    const cuuint64_t qstr[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(p.nq) * D * 2};
    const cuuint32_t qbox[3] = {64, static_cast<cuuint32_t>(p.G), 1};
    if (enc(&m->q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(p.q), qdims, qstr, qbox, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  return cudaSuccess;
}

// Sequences per near-field CTA: the count that minimises the rounds of
// resident CTAs times the items (sequence, KV head) each warp serves, plus
// one item of per-CTA start-up; the grid then ends close to a whole round.
int near_rows_for(int Lc, int n_seq, int nkv, int n_sm, int per_sm) {
  int best = 16;
  long long best_cost = -1;
  for (int r = 8; r <= kNearRowsMax; ++r) {
    const long long ctas = static_cast<long long>(Lc) * ((n_seq + r - 1) / r);
    const long long slots = static_cast<long long>(std::max(1, n_sm)) * std::max(1, per_sm);
    const long long rounds = (ctas + slots - 1) / slots;
    const long long cost = rounds * ((r * nkv + NWN - 1) / NWN + 1);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best = r;
    }
  }
  return best;
}

template <typename Tin, int D>
cudaError_t launch_t(const DecodeParams& p_in, cudaStream_t s) {
  DecodeParams p = p_in;
  WinMaps maps;
  cudaError_t e = encode_win_maps(p, D, static_cast<int>(sizeof(Tin)), &maps);
  if (e != cudaSuccess) return e;
  {
    int dev = 0, n_sm = 0, per_sm = 1;
    e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess) {
      if constexpr (sizeof(Tin) == 2)
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_near_mma_kernel<D>, NTN, p.tp.near_smem);
      else
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, decode_near_kernel<Tin, D>, NTN, p.tp.near_smem);
    }
    if (e != cudaSuccess) return e;
    p.tp.near_rows = near_rows_for(p.Lc, p.n_seq, p.nkv, n_sm, per_sm);
  }
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(p.Lc * ((p.n_seq + p.tp.near_rows - 1) / p.tp.near_rows)), 1, 1);
  cfg.blockDim = dim3(NTN, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(p.tp.near_smem);
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if constexpr (sizeof(Tin) == 2) {
    e = cudaLaunchKernelEx(&cfg, decode_near_mma_kernel<D>, p, maps);
  } else {
    e = cudaLaunchKernelEx(&cfg, decode_near_kernel<Tin, D>, p, maps);
  }
  if (e != cudaSuccess) return e;
  cfg.gridDim = dim3(static_cast<unsigned>(p.Lc * ((p.n_seq + TR - 1) / TR) * kPair), 1, 1);
  cfg.blockDim = dim3(NTP, 1, 1);  // compute warps + the MMA warp; clusters of kPair
  cfg.dynamicSmemBytes = static_cast<size_t>(p.tp.pool_smem);
  return cudaLaunchKernelEx(&cfg, decode_pool_kernel, p);
}

}  // namespace

bool plan_decode_tile(int H, int D, int esz, int G, int K, size_t limit, TilePlan* out) {
  if (H % kBlk != 0 || K < 1 || G < 1 || G > HB) return false;
  TilePlan p;
  std::memset(&p, 0, sizeof(p));
  p.pool_smem = PoolTilePlan::total + 128;  // 128: base alignment slack
  if (static_cast<size_t>(p.pool_smem) > limit) return false;
  p.near_warps = NWN;
  p.near_rows = 16;  // replaced per launch (near_rows_for)
  p.hq = 0;
  p.hkt = G * D * esz;
  p.hvt = p.hkt + D * esz;
  p.hs = p.hvt + D * esz;
  p.hdr_bytes = a128(p.hs + 4LL * D);
  if (esz == 2) {  // warp-MMA near field: fixed layout, chunks of 16 slots
    p.kcb = std::min(KCB, K);
    p.warp_bytes = D == 64 ? MmaNear<64>::warp : MmaNear<128>::warp;
    p.near_smem = 2048 + NWN * p.warp_bytes;  // barriers (1 KB) + 1 KB alignment slack
    if (static_cast<size_t>(p.near_smem) > limit) return false;
    *out = p;
    return true;
  }
  // Window chunks of 16 slots, fewer where a plan of 16 does not fit.
  for (int kcb = std::min(KCB, K); kcb >= 1; kcb /= 2) {
    p.kcb = kcb;
    p.chunk_bytes = a128(2LL * kcb * D * esz);
    p.warp_bytes = 2 * p.hdr_bytes + 2 * p.chunk_bytes;
    p.near_smem = kNearBarBytes + kNearPbBytes + NWN * p.warp_bytes + 128;
    if (static_cast<size_t>(p.near_smem) <= limit) {
      *out = p;
      return true;
    }
  }
  return false;
}

cudaError_t decode_tile_prepare(int device) {
  int optin = 0;
  cudaError_t e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, device);
  if (e == cudaSuccess) e = set_smem_t(decode_near_kernel<float, 64>, optin);
  if (e == cudaSuccess) e = set_smem_t(decode_near_kernel<float, 128>, optin);
  if (e == cudaSuccess) e = set_smem_t(decode_near_mma_kernel<64>, optin);
  if (e == cudaSuccess) e = set_smem_t(decode_near_mma_kernel<128>, optin);
  if (e == cudaSuccess) e = set_smem_t(decode_pool_kernel, optin);
  return e;
}

cudaError_t launch_decode_tile(const DecodeParams& p, int in_dtype, int head_dim, cudaStream_t s) {
  if (in_dtype == SFA_F32) return head_dim == 64 ? launch_t<float, 64>(p, s) : launch_t<float, 128>(p, s);
  return head_dim == 64 ? launch_t<__nv_bfloat16, 64>(p, s) : launch_t<__nv_bfloat16, 128>(p, s);
}

}  // namespace sfa
