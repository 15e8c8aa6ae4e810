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
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstring>

#include "sfa_common.cuh"
#include "sfa_umma.cuh"

namespace sfa {
namespace {

constexpr int NTN = 256;                // near-field kernel threads
constexpr int NWN = NTN / 32;
constexpr int HB = kDecodeTileHeads;    // query heads per KV head served
constexpr int KCB = kDecodeTileChunk;   // window slots per chunk
constexpr int kPbFloats = HB * KCB + 2 * HB;  // per warp: P, corrections, denominators
constexpr int kNearRows = 16;           // sequences per near-field CTA
static_assert(HB <= 8 && KCB == 16, "near-field lane mapping: 2 x 16 lanes, 4 heads each");

// Tensor maps of the state's window rings (keys, values) for one call:
// (head dim, KV head, slot, stream) views with boxes of one KV head x kcb
// slots.
struct WinMaps {
  CUtensorMap k, v;
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
  const int blocks_per_layer = (p.n_seq + kNearRows - 1) / kNearRows;
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
  __shared__ long long s_st[kNearRows], s_pos[kNearRows];

  if (lane == 0) {
    for (int i = 0; i < 4; ++i) mbar_init(bars + i, 1);
    mbar_fence_init();
  }
  pdl_trigger();
  pdl_wait();  // state and inputs may be written by the previous kernel
  if (tid < kNearRows) {  // the block's sequences: stream index and position
    const int bi = rb * kNearRows + tid;
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
  const int n_items = kNearRows * nkv;
  const long long in_row0 = static_cast<long long>(li) * p.n_seq + static_cast<long long>(rb) * kNearRows;
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

// ---------------------------------------------------------------- pool kernel

constexpr int NTP = 256;
constexpr int NWP = NTP / 32;
constexpr int TR = 16;                  // sequences per pool CTA (rows of the MMAs' M = 64)
constexpr int kSlotStages = 3;
constexpr int kScStride = kSlots + 1;
constexpr int kSemStride = kBlk + 4;
constexpr int kTmemCols = 256;          // scores (64) + two 64-column sem buffers
static_assert(TR * 16 == NTP, "pool kernel: 16 threads per row, 4 columns each");

// Pool CTA shared memory (byte offsets).
struct PoolTilePlan {
  static constexpr int bars = 0;                                  // mbarriers, tmem address
  static constexpr int a = 256;                                   // [2][hi, lo] x blocks
  static constexpr int w = a + 2 * 2 * kBlkBytes;                 // [hi, lo] weight block
  static constexpr int sl = w + 2 * kBlkBytes;                    // [3][hi, lo] slot blocks
  static constexpr int sc = sl + kSlotStages * 2 * kBlkBytes;     // [16][65] scores, then
  static constexpr int sem = sc;                                  // [16][68] sem chunk
  static constexpr int total = sc + TR * kSemStride * 4;
};
static_assert(TR * kScStride <= TR * kSemStride, "scores fit the sem staging");
// barrier slots
constexpr int kPbSlFull = 0;                         // [3] slot block landed
constexpr int kPbSlEmpty = kPbSlFull + kSlotStages;  // [3] MMAs done with the slot block
constexpr int kPbAEmpty = kPbSlEmpty + kSlotStages;  // [2] MMAs done with the x block
constexpr int kPbSem = kPbAEmpty + 2;                // [2] sem MMAs done
constexpr int kPbScores = kPbSem + 2;                // all score MMAs done
constexpr int kPbCount = kPbScores + 1;
static_assert(kPbCount * 8 + 4 <= PoolTilePlan::a, "barriers fit");

__global__ void __launch_bounds__(NTP, 2) decode_pool_kernel(const __grid_constant__ DecodeParams p) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int tiles_per_layer = (p.n_seq + TR - 1) / TR;
  const int li = static_cast<int>(blockIdx.x) / tiles_per_layer;
  const int tb = static_cast<int>(blockIdx.x) % tiles_per_layer;
  const int l = p.l0 + li;
  const int nch = p.H / kBlk;
  extern __shared__ __align__(128) unsigned char smb_raw[];
  unsigned char* sm = aligned128(smb_raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + PoolTilePlan::bars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kPbCount);
  unsigned char* ablk = sm + PoolTilePlan::a;
  unsigned char* wblk = sm + PoolTilePlan::w;
  unsigned char* slb = sm + PoolTilePlan::sl;
  float* sc = reinterpret_cast<float*>(sm + PoolTilePlan::sc);
  float* semc = reinterpret_cast<float*>(sm + PoolTilePlan::sem);
  __shared__ long long s_st[TR], s_pos[TR];
  __shared__ float s_ssq[TR];
  __shared__ int s_ok;

  const unsigned char* img_l = p.slot_img + static_cast<size_t>(l) * nch * 2 * kBlkBytes;
  // Slot block loads q = 0 .. 2*nch-1 (pass 1, then pass 2) through the
  // three stages: load q is block q % nch in stage q % 3.
  auto issue_slot = [&](int q) {  // tid 0
    const int st = q % kSlotStages;
    mbar_arrive_expect_tx(bars + kPbSlFull + st, 2u * kBlkBytes);
    bulk_g2s(slb + st * 2 * kBlkBytes, img_l + static_cast<size_t>(q % nch) * 2 * kBlkBytes, 2u * kBlkBytes,
             bars + kPbSlFull + st);
  };
  bool ok_slot = true;
  // After the MMAs of load q are issued: the stage of load q-1 (its MMAs
  // committed one chunk earlier) takes load q+2.  tid 0.
  auto refill_slot = [&](int q) {
    if (q < 1 || q + kSlotStages - 1 >= 2 * nch) return;
    const int st = (q - 1) % kSlotStages;
    if (!mbar_wait_bounded(bars + kPbSlEmpty + st, static_cast<unsigned>(((q - 1) / kSlotStages) & 1), kMbarPollLimit,
                           p.err))
      ok_slot = false;
    issue_slot(q + kSlotStages - 1);
  };
  if (tid == 0) {
    for (int i = 0; i < kPbCount; ++i) mbar_init(bars + i, 1);
    mbar_fence_init();
    // the slot blocks are constant since sfa_init: the first loads go out
    // before the wait for the previous kernel
    for (int q = 0; q < kSlotStages && q < 2 * nch; ++q) issue_slot(q);
  }
  if (warp == 0) tmem_alloc(tmem_slot, kTmemCols);  // at most two CTAs per SM: never waits
  // rows 16..63 of the x and weight blocks stay zero
  for (int i = tid; i < (2 * 2 + 2) * kBlkBytes / 16; i += NTP) {
    const int bi = i / (kBlkBytes / 16), rem = i % (kBlkBytes / 16);
    unsigned char* base = (bi < 4 ? ablk + bi * kBlkBytes : wblk + (bi - 4) * kBlkBytes);
    reinterpret_cast<uint4*>(base)[rem] = make_uint4(0u, 0u, 0u, 0u);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_trigger();
  pdl_wait();  // x from decode_near_kernel; the state

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
  bool ok = s_ok != 0;  // a mismatch was latched by decode_near_kernel

  // Thread tid: row r = tid / 16, columns c4 .. c4+3 of every chunk.
  const int r = tid >> 4, c4 = (tid & 15) * 4;
  const long long st = s_st[r];
  const long long io = static_cast<long long>(li) * p.n_seq + static_cast<long long>(tb) * TR + r;
  const bool live = st >= 0 && ok;
  const float* xrow = p.out + (live ? io : 0) * p.H + c4;
  auto load_x = [&](int c) -> float4 {
    return live ? __ldcg(reinterpret_cast<const float4*>(xrow + c * kBlk)) : make_float4(0.f, 0.f, 0.f, 0.f);
  };

  // ---- pass 1: scores[16 x 64] = x . slot^T and |x|^2 ----------------------
  const uint32_t idesc_s = umma_idesc_bf16(kBlk, kSlots, false);
  float4 xn0 = load_x(0);  // chunks c and c+1 in flight
  float4 xn1 = nch > 1 ? load_x(1) : make_float4(0.f, 0.f, 0.f, 0.f);
  float sq = 0.f;
  for (int c = 0; c < nch; ++c) {
    const int b = c & 1;
    const float4 v = xn0;
    xn0 = xn1;
    if (c + 2 < nch) xn1 = load_x(c + 2);
    sq = fmaf(v.x, v.x, fmaf(v.y, v.y, fmaf(v.z, v.z, fmaf(v.w, v.w, sq))));
    // x block b was read by the MMAs of chunk c-2
    if (c >= 2 && !mbar_wait_bounded(bars + kPbAEmpty + b, static_cast<unsigned>(((c - 2) >> 1) & 1), kMbarPollLimit, p.err))
      ok = false;
    unsigned char* xhi = ablk + b * 2 * kBlkBytes;
    {
      __nv_bfloat16 hh[4], ll[4];
      split_bf16(v.x, hh[0], ll[0]);
      split_bf16(v.y, hh[1], ll[1]);
      split_bf16(v.z, hh[2], ll[2]);
      split_bf16(v.w, hh[3], ll[3]);
      const int off = blk_off(r, c4);
      *reinterpret_cast<uint2*>(xhi + off) = *reinterpret_cast<const uint2*>(hh);
      *reinterpret_cast<uint2*>(xhi + kBlkBytes + off) = *reinterpret_cast<const uint2*>(ll);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      const int stg = c % kSlotStages;
      if (!mbar_wait_bounded(bars + kPbSlFull + stg, static_cast<unsigned>((c / kSlotStages) & 1), kMbarPollLimit, p.err))
        ok = false;
      tc_fence_after();
      const unsigned char* shi = slb + stg * 2 * kBlkBytes;
#pragma unroll
      for (int k = 0; k < kBlk / 16; ++k) {
        const uint64_t ah = umma_desc(xhi + k * 2048, 1024, 128), al = umma_desc(xhi + kBlkBytes + k * 2048, 1024, 128);
        const uint64_t bh = umma_desc(shi + k * 2048, 1024, 128), bl = umma_desc(shi + kBlkBytes + k * 2048, 1024, 128);
        umma_bf16(tmem, ah, bh, idesc_s, c > 0 || k > 0);
        umma_bf16(tmem, ah, bl, idesc_s, true);
        umma_bf16(tmem, al, bh, idesc_s, true);
      }
      umma_commit(bars + kPbAEmpty + b);
      umma_commit(bars + kPbSlEmpty + stg);
      refill_slot(c);
    }
  }
  if (tid == 0) umma_commit(bars + kPbScores);
  // |x|^2 per row: the 16 threads of a row (one half-warp) add their partials
#pragma unroll
  for (int off = 8; off > 0; off >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, off);
  if ((tid & 15) == 0) s_ssq[r] = sq;
  if (!mbar_wait_bounded(bars + kPbScores, 0, kMbarPollLimit, p.err)) ok = false;
  tc_fence_after();
  if ((warp & 3) == 0) {  // rows 0..15 sit in lanes 0..15 of the first lane quarter (M = 64)
    const int colh = (warp >> 2) * 32;
    float v[32];
    tmem_ld32(tmem + colh, v);
    if (lane < TR) {
#pragma unroll
      for (int jj = 0; jj < 32; ++jj) sc[lane * kScStride + colh + jj] = v[jj];
    }
  }
  tc_fence_before();
  __syncthreads();

  // ---- softmax(cos/T) per row [P3 §2.1 channel 3]; weights as split bf16 ---
  {
    const float* nrm = p.slot_norm + static_cast<size_t>(l) * kSlots;
    const float n0 = nrm[lane], n1 = nrm[lane + 32];
    for (int rr = warp; rr < TR; rr += NWP) {
      const float nx = fmaxf(sqrtf(s_ssq[rr]), kNormFloor);
      const float c0 = sc[rr * kScStride + lane] / (nx * n0) * p.inv_temp;
      const float c1 = sc[rr * kScStride + lane + 32] / (nx * n1) * p.inv_temp;
      const float mx = warp_max_redux(fmaxf(c0, c1));
      const float e0 = expf(c0 - mx), e1 = expf(c1 - mx);
      const float inv = 1.f / warp_sum(e0 + e1);
      __nv_bfloat16 h0, l0, h1, l1;
      split_bf16(e0 * inv, h0, l0);
      split_bf16(e1 * inv, h1, l1);
      const int o0 = blk_off(rr, lane), o1 = blk_off(rr, lane + 32);
      *reinterpret_cast<__nv_bfloat16*>(wblk + o0) = h0;
      *reinterpret_cast<__nv_bfloat16*>(wblk + kBlkBytes + o0) = l0;
      *reinterpret_cast<__nv_bfloat16*>(wblk + o1) = h1;
      *reinterpret_cast<__nv_bfloat16*>(wblk + kBlkBytes + o1) = l1;
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();

  // ---- pass 2: sem chunk c [16 x 64] = w . slot_c on the tensor cores; ring,
  // field, fusion, clip, output [P3 §2.1 channels 1-2, §2.2]
  const uint32_t idesc_c = umma_idesc_bf16(kBlk, kBlk, true);
  auto issue_sem = [&](int c) {  // tid 0: slot load nch + c
    const int q = nch + c, stg = q % kSlotStages;
    if (!mbar_wait_bounded(bars + kPbSlFull + stg, static_cast<unsigned>((q / kSlotStages) & 1), kMbarPollLimit, p.err))
      ok = false;
    tc_fence_after();
    const uint32_t dst = tmem + kSlots + (c & 1) * kBlk;
    const unsigned char* shi = slb + stg * 2 * kBlkBytes;
#pragma unroll
    for (int k = 0; k < kSlots / 16; ++k) {
      const uint64_t ah = umma_desc(wblk + k * 2048, 1024, 128), al = umma_desc(wblk + kBlkBytes + k * 2048, 1024, 128);
      const uint64_t bh = umma_desc(shi + k * 256, 128, 1024), bl = umma_desc(shi + kBlkBytes + k * 256, 128, 1024);
      umma_bf16(dst, ah, bh, idesc_c, k > 0);
      umma_bf16(dst, ah, bl, idesc_c, true);
      umma_bf16(dst, al, bh, idesc_c, true);
    }
    umma_commit(bars + kPbSem + (c & 1));
    umma_commit(bars + kPbSlEmpty + stg);
    refill_slot(q);
  };
  if (tid == 0) {
    issue_sem(0);
    if (nch > 1) issue_sem(1);
  }
  const int slot_r = static_cast<int>(s_pos[r] & (kRing - 1));
  unsigned char* blk = p.state + kHeaderBytes + (live ? st : 0) * p.so.stride;
  float* ring_r = reinterpret_cast<float*>(blk + p.so.ring) + static_cast<size_t>(slot_r) * p.H + c4;
  float* rsum_r = reinterpret_cast<float*>(blk + p.so.ring_sum) + c4;
  float* fld_r = reinterpret_cast<float*>(blk + p.so.field) + c4;
  float* out_r = p.out + (live ? io : 0) * p.H + c4;
  // x and state of chunks c and c+1 in flight
  struct Row4 {
    float4 x, old, rs, fl;
  };
  auto load_row = [&](int c) -> Row4 {
    Row4 v;
    if (live && c < nch) {
      v.x = __ldcg(reinterpret_cast<const float4*>(out_r + c * kBlk));
      v.old = __ldcg(reinterpret_cast<const float4*>(ring_r + c * kBlk));
      v.rs = __ldcg(reinterpret_cast<const float4*>(rsum_r + c * kBlk));
      v.fl = __ldcg(reinterpret_cast<const float4*>(fld_r + c * kBlk));
    } else {
      v.x = v.old = v.rs = v.fl = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    return v;
  };
  Row4 rn0 = load_row(0), rn1 = load_row(1);
  const float a_l = p.alpha_layer[l];
  for (int c = 0; c < nch; ++c) {
    const int b = c & 1;
    if (!mbar_wait_bounded(bars + kPbSem + b, static_cast<unsigned>((c >> 1) & 1), kMbarPollLimit, p.err)) ok = false;
    tc_fence_after();
    if ((warp & 3) == 0) {
      const int colh = (warp >> 2) * 32;
      float v[32];
      tmem_ld32(tmem + kSlots + b * kBlk + colh, v);
      if (lane < TR) {
        float* dst = semc + lane * kSemStride + colh;
#pragma unroll
        for (int jj = 0; jj < 32; jj += 4)
          *reinterpret_cast<float4*>(dst + jj) = make_float4(v[jj], v[jj + 1], v[jj + 2], v[jj + 3]);
      }
    }
    tc_fence_before();
    __syncthreads();
    if (tid == 0 && c + 2 < nch) issue_sem(c + 2);  // its buffer was read just above
    const float4 x = rn0.x, ro = rn0.old, rs = rn0.rs, fl = rn0.fl;
    const float4 sv = *reinterpret_cast<const float4*>(semc + r * kSemStride + c4);
    rn0 = rn1;
    rn1 = load_row(c + 2);
    if (live && ok) {
      const float xa[4] = {x.x, x.y, x.z, x.w}, roa[4] = {ro.x, ro.y, ro.z, ro.w};
      const float rsa[4] = {rs.x, rs.y, rs.z, rs.w}, fla[4] = {fl.x, fl.y, fl.z, fl.w};
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
      *reinterpret_cast<float4*>(ring_r + c * kBlk) = x;
      *reinterpret_cast<float4*>(rsum_r + c * kBlk) = make_float4(rv[0], rv[1], rv[2], rv[3]);
      *reinterpret_cast<float4*>(fld_r + c * kBlk) = make_float4(fv[0], fv[1], fv[2], fv[3]);
      *reinterpret_cast<float4*>(out_r + c * kBlk) = make_float4(ov[0], ov[1], ov[2], ov[3]);
    }
    __syncthreads();  // semc is rewritten by the next chunk
  }
  if (!ok_slot) ok = false;  // tid 0's waits
  if (live && ok && (tid & 15) == 0)
    *reinterpret_cast<long long*>(p.state + kHeaderBytes + st * p.so.stride + p.so.pos) = s_pos[r] + 1;

  // every tensor-core operation has completed (last sem commit waited)
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
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(p.Lc * ((p.n_seq + kNearRows - 1) / kNearRows)), 1, 1);
  cfg.blockDim = dim3(NTN, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(p.tp.near_smem);
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, decode_near_kernel<Tin, D>, p, maps);
  if (e != cudaSuccess) return e;
  cfg.gridDim = dim3(static_cast<unsigned>(p.Lc * ((p.n_seq + TR - 1) / TR)), 1, 1);
  cfg.blockDim = dim3(NTP, 1, 1);
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
  p.near_rows = kNearRows;
  p.hq = 0;
  p.hkt = G * D * esz;
  p.hvt = p.hkt + D * esz;
  p.hs = p.hvt + D * esz;
  p.hdr_bytes = a128(p.hs + 4LL * D);
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
  if (e == cudaSuccess) e = set_smem_t(decode_near_kernel<__nv_bfloat16, 64>, optin);
  if (e == cudaSuccess) e = set_smem_t(decode_near_kernel<__nv_bfloat16, 128>, optin);
  if (e == cudaSuccess) e = set_smem_t(decode_pool_kernel, optin);
  return e;
}

cudaError_t launch_decode_tile(const DecodeParams& p, int in_dtype, int head_dim, cudaStream_t s) {
  if (in_dtype == SFA_F32) return head_dim == 64 ? launch_t<float, 64>(p, s) : launch_t<float, 128>(p, s);
  return head_dim == 64 ? launch_t<__nv_bfloat16, 64>(p, s) : launch_t<__nv_bfloat16, 128>(p, s);
}

}  // namespace sfa
