// sfa_decode_tile.cu — SFA decode step for large batches: one cluster per
// (layer, tile of 64 sequences), every state update in place.
//
// Sources (web pages):
//   [P1] "Signal Field Attention (SFA)：8KB代码实现4.16倍推理加速与248倍内存压缩"
//        §2.1 eqs. O_near, S_t, O; §2.2 O(k·d) window state.
//   [P3] "Dalin Soma SFA基于信号场注意力机制的神经网络推理加速框架"
//        §2.1 channels 1–3, §2.2 fusion, clip and alpha_layer, §2.4 ring mean.
//
// At a batch of hundreds the per-stream decode kernel is bound by its chain
// of dependent memory round trips and stages a layer's slot slice once per
// sequence.  Here the 64 sequences of a tile share one cluster of CS CTAs.
//
//  * Near field [P1 §2.1 eq. O_near] and far field [eq. S_t], by KV head.
//    The work items are (sequence, KV head, block of at most 8 of its query
//    heads), spread over the cluster's CTAs, so each window is read once.
//    A copy warp streams an item's window in chunks of 16 slots (tensor
//    copies of the state's window ring) through a ring of stages, and its q
//    rows, K_t, V_t and S into a header of the warp that serves the item,
//    all counted in bytes on mbarriers.  Eight compute warps run an online
//    softmax over the chunks and P·V on the CUDA cores, then write
//    x = O_near + alpha_far·S [eq. O] of every head straight into the x tile
//    of the CTA that owns the head (distributed shared memory).
//  * Pool [P3 §2.1 channel 3]: CTA `rank` owns hidden slice [rank*HS,
//    (rank+1)*HS), HS = HPC*head_dim.  scores[64 x 64] = x . slot^T and
//    sem[64 x HS] = w . slot run on the tcgen05 tensor cores, three bf16
//    MMAs of split operands each (hi*hi + hi*lo + lo*hi, about 16
//    significant bits) accumulated in fp32 in tensor memory; the partial
//    scores and |x|^2 are summed across the cluster in distributed shared
//    memory.
//  * Ring, field, fusion, clip and output [P3 §2.1, §2.2] per element of
//    the slice.
//
// Phases:
//   (1) the tile's sequences and positions;
//   (2) near field and x (copy warp + compute warps), then a cluster
//       barrier: every x row is in place and every read of a window is done;
//   (3) write-back of the window slot and S of the items with head block 0,
//       and of the positions;
//   (4) pool scores on the tensor cores, partial sums over the slice;
//   (5) cluster reduce-scatter of the partials, softmax(cos/T), weights into
//       every CTA's shared memory;
//   (6) semantic mix on the tensor cores, then ring, field, fusion, output.
// Every wait is bounded; a wait that runs out latches SFA_ERR_DEVICE_TIMEOUT.
#include <cooperative_groups.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstring>
#include <type_traits>

#include "sfa_common.cuh"
#include "sfa_umma.cuh"

namespace cg = cooperative_groups;

namespace sfa {
namespace {

constexpr int NT = kDecodeTileThreads;  // compute threads
constexpr int NW = NT / 32;             // compute warps
constexpr int NTP = NT + 32;            // plus the copy warp
constexpr int NWP = NTP / 32;
constexpr int TB = kBlk;                // sequences per tile: the M of the pool MMAs
constexpr int HB = kDecodeTileHeads;    // query heads per near-field item
constexpr int KCB = kDecodeTileChunk;   // window slots per chunk
constexpr int kPartStride = kSlots + 1;  // 64 partial dots + |x|^2 per sequence
constexpr int kCW = kBlk;                // columns per sem chunk
constexpr int kSemStride = kCW + 4;
constexpr int kTmemCols = 256;           // scores (64) + two 64-column sem buffers
constexpr int kEpt = TB * kCW / NT;      // epilogue elements per compute thread and chunk
constexpr int kPbFloats = HB * KCB + 2 * HB;  // per warp: P, corrections, denominators
static_assert(HB <= 8 && KCB == 16, "near-field lane mapping: 2 x 16 lanes, 4 heads each");

// mbarrier slots
constexpr int kBarFull = 0;                                    // [stages] chunk landed
constexpr int kBarEmpty = kBarFull + kDecodeTileMaxStages;     // [stages] chunk consumed
constexpr int kBarHdrFull = kBarEmpty + kDecodeTileMaxStages;  // [NW] header landed
constexpr int kBarHdrEmpty = kBarHdrFull + NW;                 // [NW] header consumed
constexpr int kBarSl = kBarHdrEmpty + NW;                      // slot blocks
constexpr int kBarMs = kBarSl + 1;                             // score MMAs done with the x block
constexpr int kBarSd = kBarMs + 1;                             // all score MMAs done
constexpr int kBarMc = kBarSd + 1;                             // [2] sem MMAs done
constexpr int kNumBars = kBarMc + 2;
constexpr int kBarBytes = ((kNumBars * 8 + 16 + 127) / 128) * 128;  // + tmem address, flags

// Tensor maps of the state's window rings (keys, values) for one call:
// (head dim, KV head, slot, stream) views with boxes of one KV head x kcb
// slots.
struct WinMaps {
  CUtensorMap k, v;
};

__host__ __device__ inline int a128(long long x) { return static_cast<int>((x + 127) & ~127LL); }

template <typename Tin, int D>
__global__ void __launch_bounds__(NTP, 1)
decode_tile_kernel(const __grid_constant__ DecodeParams p, const __grid_constant__ WinMaps maps) {
  constexpr int ESZ = static_cast<int>(sizeof(Tin));
  constexpr int VE = Load16<Tin>::N;  // elements per 16-byte load
  constexpr int NC16 = D / VE;        // 16-byte chunks of one head row
  constexpr int DPL = D / 32;         // head dims per lane in P·V
  static_assert((NC16 & (NC16 - 1)) == 0, "row chunks must be a power of two");
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = static_cast<int>(cluster.block_rank());
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const TilePlan& pl = p.tp;
  const int HPC = p.HPC, HS = HPC * D, XS = HS + 4, nch = HS / kBlk;
  const int K = p.K, G = p.G, nkv = p.nkv, CS = p.CS;
  const int tiles_per_layer = (p.n_seq + TB - 1) / TB;
  const int ti = static_cast<int>(blockIdx.x) / CS;
  const int li = ti / tiles_per_layer, tb = ti % tiles_per_layer;
  const int l = p.l0 + li;

  extern __shared__ __align__(128) unsigned char smb_raw[];
  // 128-byte aligned base (the plan leaves 128 bytes of slack): the same
  // offset in every CTA, so peers' addresses map one to one.
  unsigned char* sm = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smb_raw) + 127) &
                                                       ~static_cast<uintptr_t>(127));
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + pl.bars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kNumBars);
  int* s_ok = reinterpret_cast<int*>(tmem_slot + 1);
  int* s_bad = s_ok + 1;
  float* xs = reinterpret_cast<float*>(sm + pl.xs);  // [64][XS] x of the tile
  long long* rpos = reinterpret_cast<long long*>(sm + pl.rows);
  long long* rstream = rpos + TB;
  unsigned char* simg = sm + pl.sl;                      // [nch][hi, lo] slot blocks
  float* part = reinterpret_cast<float*>(sm + pl.stg);   // [64][65] pool partials (after the
  float* semc = part;                                    // near field), then the sem chunk
  unsigned char* xw = sm + pl.xw;                        // x block (hi, lo), then w block

  if (tid == 0) {
    for (int i = 0; i < kNumBars; ++i) mbar_init(bars + i, 1);
    mbar_fence_init();
    *s_bad = 0;
    // Slot blocks: constant since sfa_init, fetched before the wait below.
    const unsigned char* img =
        p.slot_img + (static_cast<size_t>(l) * (p.H / kBlk) + static_cast<size_t>(rank) * nch) * 2 * kBlkBytes;
    mbar_arrive_expect_tx(bars + kBarSl, static_cast<unsigned>(nch * 2 * kBlkBytes));
    for (int c = 0; c < nch; ++c)
      bulk_g2s(simg + c * 2 * kBlkBytes, img + static_cast<size_t>(c) * 2 * kBlkBytes, 2u * kBlkBytes,
               bars + kBarSl);
  }
  if (warp == 0) tmem_alloc(tmem_slot, kTmemCols);  // at most two CTAs per SM: never waits
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // Peers write into this CTA's shared memory only after every CTA of the
  // cluster has started: arrive now, wait before the near field.
  cluster_arrive();
  pdl_trigger();
  pdl_wait();  // state and inputs may be written by the previous kernel

  // ---- (1) the tile's sequences and their positions -----------------------
  if (tid == 0) {
    const uint4 h0v = __ldcg(reinterpret_cast<const uint4*>(p.state));
    const uint4 h1v = __ldcg(reinterpret_cast<const uint4*>(p.state + 16));
    StateHeader hd;
    reinterpret_cast<uint4*>(&hd)[0] = h0v;
    reinterpret_cast<uint4*>(&hd)[1] = h1v;
    *s_ok = (hd.magic == kMagic) & (hd.cfg_hash == p.cfg_hash) & (hd.batch == p.B) &
            (hd.n_layers == p.L);
  }
  if (tid < TB) {
    const int bi = tb * TB + tid;
    long long st = -1, ps = 0;
    if (bi < p.n_seq) {
      const int b = p.seq_ids ? __ldcg(p.seq_ids + bi) : bi;
      if (b >= 0 && b < p.B) {
        st = static_cast<long long>(l) * p.B + b;
        ps = __ldcg(reinterpret_cast<const long long*>(p.state + kHeaderBytes + st * p.so.stride + p.so.pos));
      } else if (rank == 0) {
        latch_error(p.err, SFA_ERR_INVALID_ARG);
      }
    }
    rstream[tid] = st;
    rpos[tid] = ps;
  }
  __syncthreads();
  cluster_wait();
  if (!*s_ok) {  // the same header for every CTA: the whole grid leaves here
    mbar_wait_bounded(bars + kBarSl, 0, kMbarPollLimit, p.err);  // no copy may land after exit
    if (tid == 0 && rank == 0 && ti == 0) latch_error(p.err, SFA_ERR_STATE_MISMATCH);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
      tc_fence_after();
      tmem_dealloc(tmem, kTmemCols);
    }
    return;
  }
  for (int idx = tid; idx < TB * HS; idx += NTP)  // rows without a sequence stay zero
    if (rstream[idx / HS] < 0) xs[(idx / HS) * XS + idx % HS] = 0.f;

  // ---- (2) near field, far field, x -------------------------------------
  // Item it = rank + m*CS (m = 0, 1, ...) of this CTA is row it / per_row,
  // KV head g and head block hb of the rest; its chunks are m*nck ..
  // m*nck + nck - 1 in the copy order, chunk c in stage c % ns.
  const int nhb = (G + HB - 1) / HB;
  const int per_row = nkv * nhb;
  const int n_items = TB * per_row;
  const int n_my = rank < n_items ? (n_items - 1 - rank) / CS + 1 : 0;
  const int kcb = pl.kcb;
  const int nck = (K + kcb - 1) / kcb;
  const int NS = pl.ns;
  const long long in_row0 = static_cast<long long>(li) * p.n_seq + static_cast<long long>(tb) * TB;
  if (warp == NW) {
    // Copy warp: one lane issues every copy of the CTA's items in order.
    if (lane == 0) {
      bool ok = true;
      const int total = n_my * nck;
      for (int c = 0; c < total; ++c) {
        const int m = c / nck, piece = c - m * nck;
        const int it = rank + m * CS;
        const int r = it / per_row, rem = it - r * per_row, g = rem / nhb, hb = rem - g * nhb;
        const int h0 = g * G + hb * HB, nh = min(HB, G - hb * HB);
        const long long st = rstream[r];
        const long long io = in_row0 + r;  // input row
        if (piece == 0) {
          const int w = m % NW;
          uint64_t* hf = bars + kBarHdrFull + w;
          // the warp's previous item has released the header
          if (m >= NW && !mbar_wait_bounded(bars + kBarHdrEmpty + w, static_cast<unsigned>(((m / NW) - 1) & 1),
                                            kMbarPollLimit, p.err))
            ok = false;
          unsigned char* hd = sm + pl.hdr + w * pl.hdr_bytes;
          if (st >= 0) {
            mbar_arrive_expect_tx(hf, static_cast<unsigned>((nh + 2) * D * ESZ + 4 * D));
            bulk_g2s(hd + pl.hq, static_cast<const Tin*>(p.q) + (io * p.nq + h0) * D,
                     static_cast<unsigned>(nh * D * ESZ), hf);
            bulk_g2s(hd + pl.hkt, static_cast<const Tin*>(p.k) + (io * nkv + g) * D, D * ESZ, hf);
            bulk_g2s(hd + pl.hvt, static_cast<const Tin*>(p.v) + (io * nkv + g) * D, D * ESZ, hf);
            bulk_g2s(hd + pl.hs, p.state + kHeaderBytes + st * p.so.stride + p.so.far + static_cast<long long>(g) * D * 4,
                     D * 4, hf);
          } else {
            mbar_arrive(hf);
          }
        }
        const int si = c % NS;
        if (c >= NS && !mbar_wait_bounded(bars + kBarEmpty + si, static_cast<unsigned>(((c / NS) - 1) & 1),
                                          kMbarPollLimit, p.err))
          ok = false;
        unsigned char* sg = sm + pl.stg + si * pl.stage;
        if (st >= 0) {
          mbar_arrive_expect_tx(bars + kBarFull + si, static_cast<unsigned>(2 * kcb * D * ESZ));
          tma_load_4d(sg, &maps.k, 0, g, piece * kcb, static_cast<int>(st), bars + kBarFull + si);
          tma_load_4d(sg + kcb * D * ESZ, &maps.v, 0, g, piece * kcb, static_cast<int>(st), bars + kBarFull + si);
        } else {
          mbar_arrive(bars + kBarFull + si);
        }
      }
      if (!ok) *s_bad = 1;
    }
  } else {
    // Compute warps.  QK: lane (j, half) scores chunk slot j against the
    // item's heads half, half+2, half+4, half+6; each lane starts its walk
    // along the head row at 16-byte chunk j, so the lanes of a half hit
    // distinct banks.  P·V: lane owns head dims lane*DPL .. +DPL of every
    // head.
    float* pbw = reinterpret_cast<float*>(sm + pl.pb) + warp * kPbFloats;
    float* pP = pbw;                // [HB][KCB] softmax numerators of the chunk
    float* pCorr = pbw + HB * KCB;  // [HB] rescale of the running sums
    float* pDen = pCorr + HB;       // [HB] final denominators
    const unsigned char* hd = sm + pl.hdr + warp * pl.hdr_bytes;
    const Tin* qh = reinterpret_cast<const Tin*>(hd + pl.hq);
    const Tin* ktr = reinterpret_cast<const Tin*>(hd + pl.hkt);
    const Tin* vtr = reinterpret_cast<const Tin*>(hd + pl.hvt);
    const float* s_old = reinterpret_cast<const float*>(hd + pl.hs);
    const int j = lane & 15, half = lane >> 4, d0 = lane * DPL;
    bool ok = true;
    for (int m = warp; m < n_my; m += NW) {
      const int it = rank + m * CS;
      const int r = it / per_row, rem = it - r * per_row, g = rem / nhb, hb = rem - g * nhb;
      const int h0 = g * G + hb * HB, nh = min(HB, G - hb * HB);
      const long long st = rstream[r];
      const long long t = rpos[r];
      const int es = static_cast<int>(t % K);  // slot of token t: holds the evicted key t-k
      const bool full_win = t >= K - 1;        // every slot holds a position >= 0
      if (!mbar_wait_bounded(bars + kBarHdrFull + warp, static_cast<unsigned>((m / NW) & 1), kMbarPollLimit, p.err))
        ok = false;
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
      for (int piece = 0; piece < nck; ++piece) {
        const int c = m * nck + piece;
        const int si = c % NS;
        if (!mbar_wait_bounded(bars + kBarFull + si, static_cast<unsigned>((c / NS) & 1), kMbarPollLimit, p.err))
          ok = false;
        const Tin* kc = reinterpret_cast<const Tin*>(sm + pl.stg + si * pl.stage);
        const Tin* vc = kc + kcb * D;
        if (st >= 0) {
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
                if (half + 2 * u < nh) {
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
            if (hh < nh) {
              pP[hh * KCB + j] = pj;
              if (j == 0) pCorr[hh] = corr;
            }
          }
          __syncwarp();
          // P·V over the chunk's valid slots (uniform over the warp)
#pragma unroll
          for (int hh = 0; hh < HB; ++hh) {
            if (hh < nh) {
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
              if (hh < nh) {
                const float pv = pP[hh * KCB + jj];
#pragma unroll
                for (int e = 0; e < DPL; ++e) o[hh][e] = fmaf(pv, vv[e], o[hh][e]);
              }
            }
          }
          // the key that token t evicts (the old content of slot es)
          if (piece == es / kcb) VecLoad<Tin, DPL>::run(kc + (es - piece * kcb) * D + d0, kev);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(bars + kBarEmpty + si);
      }
      if (st >= 0) {
        // x = O_near + alpha_far * S_t into the x tile of each head's owner
        if (j == 0) {
#pragma unroll
          for (int u = 0; u < 4; ++u)
            if (half + 2 * u < nh) pDen[half + 2 * u] = drun[u];
        }
        __syncwarp();
        float sn[DPL];
#pragma unroll
        for (int e = 0; e < DPL; ++e) sn[e] = (t >= K) ? ewma(p.gamma_far, s_old[d0 + e], kev[e]) : s_old[d0 + e];
#pragma unroll
        for (int hh = 0; hh < HB; ++hh) {
          if (hh < nh) {
            const float inv = 1.f / pDen[hh];
            const int h = h0 + hh, owner = h / HPC;
            float* dst = cluster.map_shared_rank(xs, owner) + r * XS + (h - owner * HPC) * D + d0;
            float v[DPL];
#pragma unroll
            for (int e = 0; e < DPL; ++e) v[e] = fmaf(p.alpha_far, sn[e], o[hh][e] * inv);
            if constexpr (DPL == 4) {
              *reinterpret_cast<float4*>(dst) = make_float4(v[0], v[1], v[2], v[3]);
            } else {
              *reinterpret_cast<float2*>(dst) = make_float2(v[0], v[1]);
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bars + kBarHdrEmpty + warp);
    }
    if (!ok) *s_bad = 1;
  }
  __syncthreads();
  cluster.sync();  // x rows of every item are in place; every window read is done

  // ---- (3) write-back of the items with head block 0: S with the evicted
  // key, K_t and V_t into slot t mod k; the positions
  if (!*s_bad) {
    for (int idx = tid; idx < n_my * D; idx += NTP) {
      const int m = idx / D, i = idx - m * D;
      const int it = rank + m * CS;
      const int r = it / per_row, rem = it - r * per_row, g = rem / nhb, hb = rem - g * nhb;
      const long long st = rstream[r];
      if (hb != 0 || st < 0) continue;
      const long long t = rpos[r];
      const long long io = in_row0 + r;
      unsigned char* blk = p.state + kHeaderBytes + st * p.so.stride;
      Tin* win_k = reinterpret_cast<Tin*>(blk + p.so.win_k);
      Tin* win_v = reinterpret_cast<Tin*>(blk + p.so.win_v);
      float* far = reinterpret_cast<float*>(blk + p.so.far);
      const size_t wo = (static_cast<size_t>(t % K) * nkv + g) * D + i;
      float s = far[g * D + i];
      if (t >= K) s = ewma(p.gamma_far, s, to_f32<Tin>(win_k[wo]));
      far[g * D + i] = s;
      win_k[wo] = static_cast<const Tin*>(p.k)[(io * nkv + g) * D + i];
      win_v[wo] = static_cast<const Tin*>(p.v)[(io * nkv + g) * D + i];
    }
    if (rank == 0 && tid < TB && rstream[tid] >= 0)
      *reinterpret_cast<long long*>(p.state + kHeaderBytes + rstream[tid] * p.so.stride + p.so.pos) = rpos[tid] + 1;
  }

  // ---- (4) pool scores on the tensor cores [P3 §2.1 channel 3] -----------
  const uint32_t idesc_s = umma_idesc_bf16(kBlk, kSlots, false);
  const uint32_t idesc_c = umma_idesc_bf16(kBlk, kCW, true);
  unsigned char* xhi = xw;
  unsigned char* xlo = xw + kBlkBytes;
  bool ok4 = true;
  for (int c = 0; c < nch; ++c) {
    if (c >= 1)  // the MMAs of chunk c-1 have finished reading the x block
      if (!mbar_wait_bounded(bars + kBarMs, (c - 1) & 1, kMbarPollLimit, p.err)) ok4 = false;
    stage_split_block(xs + c * kBlk, XS, xhi, xlo, tid, NTP);
    fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0) {
      if (c == 0 && !mbar_wait_bounded(bars + kBarSl, 0, kMbarPollLimit, p.err)) ok4 = false;
      tc_fence_after();
      const unsigned char* shi = simg + c * 2 * kBlkBytes;
      const unsigned char* slo = shi + kBlkBytes;
#pragma unroll
      for (int s2 = 0; s2 < kBlk / 16; ++s2) {
        const uint64_t ah = umma_desc(xhi + s2 * 2048, 1024, 128), al = umma_desc(xlo + s2 * 2048, 1024, 128);
        const uint64_t bh = umma_desc(shi + s2 * 2048, 1024, 128), bl = umma_desc(slo + s2 * 2048, 1024, 128);
        umma_bf16(tmem, ah, bh, idesc_s, c > 0 || s2 > 0);
        umma_bf16(tmem, ah, bl, idesc_s, true);
        umma_bf16(tmem, al, bh, idesc_s, true);
      }
      umma_commit(bars + kBarMs);
    }
  }
  if (tid == 0) umma_commit(bars + kBarSd);
  for (int r = warp; r < TB; r += NWP) {  // |x|^2 per sequence while the MMAs finish
    float ss = 0.f;
    for (int e = lane; e < HS; e += 32) ss = fmaf(xs[r * XS + e], xs[r * XS + e], ss);
    ss = warp_sum(ss);
    if (lane == 0) part[r * kPartStride + kSlots] = ss;
  }
  if (!mbar_wait_bounded(bars + kBarSd, 0, kMbarPollLimit, p.err)) ok4 = false;
  tc_fence_after();
  if (warp < NW) {  // accumulator row r sits in lane (r % 16) + 32 (r / 16) for M = 64
    const int sp = warp & 3, colh = (warp >> 2) * 32;
    float v[32];
    tmem_ld32(tmem + (static_cast<uint32_t>(32 * sp) << 16) + colh, v);
    if (lane < 16) {
      const int r = 16 * sp + lane;
#pragma unroll
      for (int jj = 0; jj < 32; ++jj) part[r * kPartStride + colh + jj] = v[jj];
    }
  }
  if (!ok4) *s_bad = 1;
  tc_fence_before();

  // ---- (5) cluster reduce-scatter of the pool sums, softmax(cos/T) -------
  cluster.sync();
  if (warp < NW) {
    const float* nrm = p.slot_norm + static_cast<size_t>(l) * kSlots;
    const float n0 = nrm[lane], n1 = nrm[lane + 32];
    for (int r = rank + CS * warp; r < TB; r += CS * NW) {
      float v0[kMaxCluster], v1[kMaxCluster], vs[kMaxCluster];
#pragma unroll
      for (int q = 0; q < kMaxCluster; ++q) {
        const bool in = q < CS;
        const float* rp = cluster.map_shared_rank(part, in ? q : 0) + r * kPartStride;
        v0[q] = in ? rp[lane] : 0.f;
        v1[q] = in ? rp[lane + 32] : 0.f;
        vs[q] = in ? rp[kSlots] : 0.f;
      }
      float s0 = 0.f, s1 = 0.f, ss = 0.f;
#pragma unroll
      for (int q = 0; q < kMaxCluster; ++q) {
        s0 += v0[q];
        s1 += v1[q];
        ss += vs[q];
      }
      const float nx = fmaxf(sqrtf(ss), kNormFloor);
      const float c0 = s0 / (nx * n0) * p.inv_temp;
      const float c1 = s1 / (nx * n1) * p.inv_temp;
      const float mx = warp_max_redux(fmaxf(c0, c1));
      const float e0 = expf(c0 - mx), e1 = expf(c1 - mx);
      const float inv = 1.f / warp_sum(e0 + e1);
      __nv_bfloat16 hb0, lb0, hb1, lb1;
      split_bf16(e0 * inv, hb0, lb0);
      split_bf16(e1 * inv, hb1, lb1);
      const int o0 = blk_off(r, lane), o1 = blk_off(r, lane + 32);
      for (int q = 0; q < CS; ++q) {
        unsigned char* wq = cluster.map_shared_rank(xw, q);  // the x blocks are dead everywhere
        *reinterpret_cast<__nv_bfloat16*>(wq + o0) = hb0;
        *reinterpret_cast<__nv_bfloat16*>(wq + kBlkBytes + o0) = lb0;
        *reinterpret_cast<__nv_bfloat16*>(wq + o1) = hb1;
        *reinterpret_cast<__nv_bfloat16*>(wq + kBlkBytes + o1) = lb1;
      }
    }
    fence_proxy_async_cluster();
  }
  cluster.sync();

  // ---- (6a) semantic mix on the tensor cores: sem chunk c [64 x 64] =
  // w . slot_chunk_c, accumulators alternating between tensor-memory columns
  // 64..127 and 128..191.
  unsigned char* whi = xw;
  unsigned char* wlo = xw + kBlkBytes;
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  auto issue_sem = [&](int c) {  // tid 0 only
    tc_fence_after();
    const uint32_t dst = tmem + kSlots + (c & 1) * kCW;
    const unsigned char* shi = simg + c * 2 * kBlkBytes;
    const unsigned char* slo = shi + kBlkBytes;
#pragma unroll
    for (int s2 = 0; s2 < kSlots / 16; ++s2) {
      const uint64_t ah = umma_desc(whi + s2 * 2048, 1024, 128), al = umma_desc(wlo + s2 * 2048, 1024, 128);
      const uint64_t bh = umma_desc(shi + s2 * 256, 128, 1024), bl = umma_desc(slo + s2 * 256, 128, 1024);
      umma_bf16(dst, ah, bh, idesc_c, s2 > 0);
      umma_bf16(dst, ah, bl, idesc_c, true);
      umma_bf16(dst, al, bh, idesc_c, true);
    }
    umma_commit(bars + kBarMc + (c & 1));
  };
  if (tid == 0) {
    issue_sem(0);
    if (nch > 1) issue_sem(1);
  }

  // ---- (6b) per sem chunk: ring, field, fusion, clip, output -------------
  // [P3 §2.1 channels 1-2, §2.2]; compute thread (row, column) elements with
  // the columns consecutive, the state values loaded before the MMA wait.
  const float a_l = p.alpha_layer[l];
  const bool write_ok = !*s_bad;
  for (int c = 0; c < nch; ++c) {
    float old_r[kEpt], rs_r[kEpt], fl_r[kEpt];
#pragma unroll
    for (int u = 0; u < kEpt; ++u) {
      old_r[u] = rs_r[u] = fl_r[u] = 0.f;
      if (tid >= NT) continue;
      const int idx = u * NT + tid, r = idx / kCW, e = c * kCW + idx % kCW;
      const long long st = rstream[r];
      if (st >= 0) {
        const unsigned char* blk = p.state + kHeaderBytes + st * p.so.stride;
        const int gi = rank * HS + e;
        old_r[u] = reinterpret_cast<const float*>(blk + p.so.ring)[static_cast<size_t>(rpos[r] & (kRing - 1)) * p.H + gi];
        rs_r[u] = reinterpret_cast<const float*>(blk + p.so.ring_sum)[gi];
        fl_r[u] = reinterpret_cast<const float*>(blk + p.so.field)[gi];
      }
    }
    const int buf = c & 1;
    bool okc = mbar_wait_bounded(bars + kBarMc + buf, (c >> 1) & 1, kMbarPollLimit, p.err);
    tc_fence_after();
    if (warp < NW) {
      const int sp = warp & 3, colh = (warp >> 2) * 32;
      float v[32];
      tmem_ld32(tmem + (static_cast<uint32_t>(32 * sp) << 16) + kSlots + buf * kCW + colh, v);
      if (lane < 16) {
        float* dst = semc + (16 * sp + lane) * kSemStride + colh;
#pragma unroll
        for (int jj = 0; jj < 32; jj += 4)
          *reinterpret_cast<float4*>(dst + jj) = make_float4(v[jj], v[jj + 1], v[jj + 2], v[jj + 3]);
      }
    }
    tc_fence_before();
    __syncthreads();
    if (tid == 0 && c + 2 < nch) issue_sem(c + 2);  // overlaps the epilogue below
    if (tid < NT && okc && write_ok) {
#pragma unroll
      for (int u = 0; u < kEpt; ++u) {
        const int idx = u * NT + tid, r = idx / kCW, cc = idx % kCW, e = c * kCW + cc;
        const long long st = rstream[r];
        if (st < 0) continue;
        unsigned char* blk = p.state + kHeaderBytes + st * p.so.stride;
        const int gi = rank * HS + e;
        const float x = xs[r * XS + e];
        const float rv = (rs_r[u] - old_r[u]) + x;       // ring sum after storing x_t
        const float fv = ewma(p.ema_gamma, fl_r[u], x);  // EMA field
        float uu = rv * (1.0f / kRing) + 0.5f * fv + 0.5f * semc[r * kSemStride + cc];
        uu = fminf(fmaxf(uu, -p.clip_eps), p.clip_eps);
        reinterpret_cast<float*>(blk + p.so.ring)[static_cast<size_t>(rpos[r] & (kRing - 1)) * p.H + gi] = x;
        reinterpret_cast<float*>(blk + p.so.ring_sum)[gi] = rv;
        reinterpret_cast<float*>(blk + p.so.field)[gi] = fv;
        const long long io = in_row0 + r;
        p.out[io * p.H + gi] = fmaf(a_l, uu, x);
      }
    }
    __syncthreads();  // semc is rewritten by the next chunk
  }

  // every tensor-core operation has completed (last sem commit waited)
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <typename Tin, int D>
cudaError_t prepare_t(int optin) {
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, decode_tile_kernel<Tin, D>);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(decode_tile_kernel<Tin, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             optin - static_cast<int>(fa.sharedSizeBytes));
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(decode_tile_kernel<Tin, D>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
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
// slot, stream) tensors; boxes of head_dim x 1 x kcb x 1.
cudaError_t encode_win_maps(const DecodeParams& p, int D, int esz, WinMaps* m) {
  PFN_cuTensorMapEncodeTiled_v12000 enc = tile_map_encoder();
  if (!enc) return cudaErrorNotSupported;
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(p.nkv),
                              static_cast<cuuint64_t>(p.K),
                              static_cast<cuuint64_t>(p.L) * static_cast<cuuint64_t>(p.B)};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(D) * esz, static_cast<cuuint64_t>(p.nkv) * D * esz,
                                 static_cast<cuuint64_t>(p.so.stride)};
  const cuuint32_t box[4] = {static_cast<cuuint32_t>(D), 1, static_cast<cuuint32_t>(p.tp.kcb), 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUtensorMapDataType dt = esz == 4 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  auto one = [&](CUtensorMap* map, long long off) -> bool {
    void* base = p.state + kHeaderBytes + off;
    return enc(map, dt, 4, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
  };
  if (!one(&m->k, p.so.win_k) || !one(&m->v, p.so.win_v)) return cudaErrorInvalidValue;
  return cudaSuccess;
}

template <typename Tin, int D>
cudaError_t launch_t(const DecodeParams& p, cudaStream_t s) {
  WinMaps maps;
  cudaError_t e = encode_win_maps(p, D, static_cast<int>(sizeof(Tin)), &maps);
  if (e != cudaSuccess) return e;
  const int tiles = p.Lc * ((p.n_seq + TB - 1) / TB);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(tiles * p.CS), 1, 1);
  cfg.blockDim = dim3(NTP, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(p.tp.total);
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = p.CS;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, decode_tile_kernel<Tin, D>, p, maps);
}

template <typename Tin, int D>
int max_clusters_t(int cs, size_t smem) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(cs * 16), 1, 1);
  cfg.blockDim = dim3(NTP, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cs;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, decode_tile_kernel<Tin, D>, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}

}  // namespace

bool plan_decode_tile(int HPC, int D, int esz, int G, int K, size_t limit, TilePlan* out) {
  const int HS = HPC * D;
  if (HS % kBlk != 0 || K < 1 || G < 1) return false;
  // Window chunks of 16 slots, fewer where a plan of 16 does not fit.
  for (int kcb = std::min(KCB, K); kcb >= 1; kcb /= 2) {
    TilePlan p;
    std::memset(&p, 0, sizeof(p));
    p.kcb = kcb;
    int o = 0;
    p.bars = o;  o += kBarBytes;
    p.xs = o;    o += a128(4LL * TB * (HS + 4));
    p.rows = o;  o += a128(16LL * TB);
    p.sl = o;    o += a128(static_cast<long long>(HS / kBlk) * 2 * kBlkBytes);
    p.xw = o;    o += 2 * kBlkBytes;
    p.pb = o;    o += a128(4LL * NW * kPbFloats);
    p.hq = 0;
    p.hkt = p.hq + std::min(HB, G) * D * esz;  // q rows of one item's heads
    p.hvt = p.hkt + D * esz;
    p.hs = p.hvt + D * esz;
    p.hdr_bytes = a128(p.hs + 4LL * D);
    p.hdr = o;   o += NW * p.hdr_bytes;
    p.stage = a128(2LL * p.kcb * D * esz);
    p.stg = o;
    // the pool partials and the sem chunk reuse the stages
    const long long reuse = std::max(4LL * TB * kPartStride, 4LL * TB * kSemStride);
    const long long avail = static_cast<long long>(limit) - 128 - o;  // 128: base alignment slack
    if (avail < 2LL * p.stage) continue;
    const int ns = static_cast<int>(std::min<long long>(kDecodeTileMaxStages, avail / p.stage));
    const long long area = std::max(static_cast<long long>(ns) * p.stage, reuse);
    if (area > avail) continue;
    p.ns = ns;
    o += static_cast<int>(area);
    // More than a third of the SM's shared memory: at most two CTAs share an
    // SM, so their tensor-memory allocations (256 columns each) always fit.
    p.total = static_cast<int>(std::max(static_cast<long long>(o) + 128,
                                        (static_cast<long long>(limit) + 1024) / 3 + 1));
    if (p.total > static_cast<long long>(limit)) continue;
    *out = p;
    return true;
  }
  return false;
}

int decode_tile_max_active_clusters(int cs, size_t smem, int in_dtype, int head_dim) {
  if (in_dtype == SFA_F32) return head_dim == 64 ? max_clusters_t<float, 64>(cs, smem) : max_clusters_t<float, 128>(cs, smem);
  return head_dim == 64 ? max_clusters_t<__nv_bfloat16, 64>(cs, smem)
                        : max_clusters_t<__nv_bfloat16, 128>(cs, smem);
}

cudaError_t decode_tile_prepare(int device) {
  int optin = 0;
  cudaError_t e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, device);
  if (e == cudaSuccess) e = prepare_t<float, 64>(optin);
  if (e == cudaSuccess) e = prepare_t<float, 128>(optin);
  if (e == cudaSuccess) e = prepare_t<__nv_bfloat16, 64>(optin);
  if (e == cudaSuccess) e = prepare_t<__nv_bfloat16, 128>(optin);
  return e;
}

cudaError_t launch_decode_tile(const DecodeParams& p, int in_dtype, int head_dim, cudaStream_t s) {
  if (in_dtype == SFA_F32) return head_dim == 64 ? launch_t<float, 64>(p, s) : launch_t<float, 128>(p, s);
  return head_dim == 64 ? launch_t<__nv_bfloat16, 64>(p, s) : launch_t<__nv_bfloat16, 128>(p, s);
}

}  // namespace sfa
