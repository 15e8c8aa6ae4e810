// sfa_decode_tile.cu — SFA decode step for large batches: one cluster per
// (layer, tile of 64 sequences), every state update in place.
//
// Sources (web pages):
//   [P1] "Signal Field Attention (SFA)：8KB代码实现4.16倍推理加速与248倍内存压缩"
//        §2.1 eqs. O_near, S_t, O; §2.2 O(k·d) window state.
//   [P3] "Dalin Soma SFA基于信号场注意力机制的神经网络推理加速框架"
//        §2.1 channels 1–3, §2.2 fusion, clip and alpha_layer, §2.4 ring mean.
//
// The per-stream decode kernel stages a layer's slot slice once per
// sequence; at a batch of hundreds that traffic (64 x hidden fp32 per
// sequence and layer) and the per-stream latency chain dominate.  Here the
// 64 sequences of a tile share one staged slot slice and the semantic pool
// becomes a matrix product with the sequences as rows, on the tensor cores
// exactly as in the prefill: scores[64 x 64] = x . slot^T and
// sem[64 x HS] = w . slot, each as three bf16 MMAs of split operands
// (hi*hi + hi*lo + lo*hi, about 16 significant bits) accumulated in fp32.
//
// CTA `rank` of the cluster owns query heads [rank*HPC, (rank+1)*HPC), i.e.
// hidden slice [rank*HS, (rank+1)*HS).  Phases:
//   (1) positions of the tile's sequences;
//   (2) near field per (sequence, head), one warp each, window rows read
//       straight from the state; far field with the evicted key; x tile;
//   (3) pool scores on the tensor cores, partial sums over the slice;
//   (4) cluster reduce-scatter of the partials, softmax(cos/T), weights into
//       every CTA's shared memory (distributed shared memory);
//   (5) write-back of the window slot and S of the KV heads this CTA owns
//       (after the cluster barrier of (4): every CTA has read them);
//   (6) semantic mix on the tensor cores, then ring, field, fusion, output.
// Every wait is bounded; a wait that runs out latches SFA_ERR_DEVICE_TIMEOUT.
#include <cooperative_groups.h>
#include <cuda_bf16.h>

#include <algorithm>
#include <type_traits>

#include "sfa_common.cuh"
#include "sfa_umma.cuh"

namespace cg = cooperative_groups;

namespace sfa {
namespace {

constexpr int NT = kDecodeTileThreads;
constexpr int NW = NT / 32;
constexpr int TB = kBlk;                 // sequences per tile: the M of the pool MMAs
constexpr int kPartStride = kSlots + 1;  // 64 partial dots + |x|^2 per sequence
constexpr int kCW = kBlk;                // columns per sem chunk
constexpr int kSemStride = kCW + 4;
constexpr int kTmemCols = 256;           // scores (64) + two 64-column sem buffers
constexpr int kEpt = TB * kCW / NT;      // epilogue elements per thread and chunk

struct TilePlan {
  int bars, xs, rows, sl, part, xw, total;
};

__host__ __device__ inline int a16t(long long x) { return static_cast<int>((x + 15) & ~15LL); }

__host__ __device__ inline TilePlan tile_plan(int HS) {
  TilePlan p;
  int o = 0;
  p.bars = o;  o += 128;
  p.xs = o;    o += a16t(4LL * TB * (HS + 4));
  p.rows = o;  o += a16t(16LL * TB);  // per row: position, stream index (-1: no sequence)
  p.sl = o;    o += a16t(static_cast<long long>(HS / kBlk) * 2 * kBlkBytes);
  p.part = o;  o += a16t(4LL * TB * (kPartStride > kSemStride ? kPartStride : kSemStride));
  p.xw = o;    o += 2 * kBlkBytes;
  p.total = o;
  return p;
}

template <typename Tin, int D>
__global__ void __launch_bounds__(NT, 1)
decode_tile_kernel(const DecodeParams p) {
  constexpr int EPL = D / 32;
  constexpr int VE = Load16<Tin>::N;
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = static_cast<int>(cluster.block_rank());
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int HPC = p.HPC, HS = HPC * D, XS = HS + 4, nch = HS / kBlk;
  const int K = p.K, G = p.G, nkv = p.nkv;
  const int h0 = rank * HPC;
  const int g_hi = (h0 + HPC - 1) / G;
  const int own_lo = (h0 + G - 1) / G;  // KV heads whose window and S this CTA writes
  const int tiles_per_layer = (p.n_seq + TB - 1) / TB;
  const int ti = static_cast<int>(blockIdx.x) / p.CS;
  const int li = ti / tiles_per_layer, tb = ti % tiles_per_layer;
  const int l = p.l0 + li;

  extern __shared__ __align__(16) unsigned char smb[];
  const TilePlan pl = tile_plan(HS);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smb + pl.bars);
  uint64_t* bar_sl = bars + 0;  // slot blocks
  uint64_t* bar_ms = bars + 1;  // score MMAs done with the x block
  uint64_t* bar_sd = bars + 2;  // all score MMAs done
  uint64_t* bar_mc = bars + 3;  // [2] sem MMAs done, per accumulator
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 8);
  float* xs = reinterpret_cast<float*>(smb + pl.xs);          // [64][XS] x of the tile
  long long* rpos = reinterpret_cast<long long*>(smb + pl.rows);
  long long* rstream = rpos + TB;
  unsigned char* simg = smb + pl.sl;                          // [nch][hi, lo] slot blocks
  float* part = reinterpret_cast<float*>(smb + pl.part);      // [64][65] pool partials, then
  float* semc = part;                                         // [64][68] the sem chunk
  unsigned char* xw = smb + pl.xw;                            // x block (hi, lo), then w block
  __shared__ int s_ok;
  __shared__ int s_bad;

  if (tid == 0) {
    for (int i = 0; i < 5; ++i) mbar_init(bars + i, 1);
    mbar_fence_init();
    s_bad = 0;
    // Slot blocks: constant since sfa_init, fetched before the wait below.
    const unsigned char* img =
        p.slot_img + (static_cast<size_t>(l) * (p.H / kBlk) + static_cast<size_t>(rank) * nch) * 2 * kBlkBytes;
    mbar_arrive_expect_tx(bar_sl, static_cast<unsigned>(nch * 2 * kBlkBytes));
    for (int c = 0; c < nch; ++c)
      bulk_g2s(simg + c * 2 * kBlkBytes, img + static_cast<size_t>(c) * 2 * kBlkBytes, 2u * kBlkBytes, bar_sl);
  }
  if (warp == 0) tmem_alloc(tmem_slot, kTmemCols);  // one CTA per SM: never waits
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_trigger();
  pdl_wait();  // state and inputs may be written by the previous kernel

  // ---- (1) the tile's sequences and their positions -----------------------
  if (tid == 0) {
    const uint4 h0v = __ldcg(reinterpret_cast<const uint4*>(p.state));
    const uint4 h1v = __ldcg(reinterpret_cast<const uint4*>(p.state + 16));
    StateHeader hd;
    reinterpret_cast<uint4*>(&hd)[0] = h0v;
    reinterpret_cast<uint4*>(&hd)[1] = h1v;
    s_ok = (hd.magic == kMagic) & (hd.cfg_hash == p.cfg_hash) & (hd.batch == p.B) &
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
  if (!s_ok) {  // the same header for every CTA: the whole grid leaves here
    mbar_wait_bounded(bar_sl, 0, kMbarPollLimit, p.err);  // no copy may land after exit
    if (tid == 0 && rank == 0 && ti == 0) latch_error(p.err, SFA_ERR_STATE_MISMATCH);
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
      tc_fence_after();
      tmem_dealloc(tmem, kTmemCols);
    }
    return;
  }
  for (int idx = tid; idx < TB * HS; idx += NT)  // rows without a sequence stay zero
    if (rstream[idx / HS] < 0) xs[(idx / HS) * XS + idx % HS] = 0.f;

  // ---- (2) near field [P1 §2.1 eq. O_near], far field [eq. S_t], x [eq. O]
  // One warp per (sequence, head): KPC window positions at a time with
  // LPK = 32/KPC lanes per position splitting the q·K dot product, online
  // softmax, P·V with lanes over head dims.
  auto near_pairs = [&](auto kpc_c) {
    constexpr int KPC = decltype(kpc_c)::value;
    constexpr int LPK = 32 / KPC;
    constexpr int DL = D / LPK;
    const int key = lane / LPK, part_l = lane % LPK;
    for (int pr = warp; pr < TB * HPC; pr += NW) {
      const int r = pr % TB, hh = pr / TB;
      const long long st = rstream[r];
      if (st < 0) continue;
      const long long t = rpos[r];
      const long long io = static_cast<long long>(li) * p.n_seq + tb * TB + r;  // input / output row
      const unsigned char* blk = p.state + kHeaderBytes + st * p.so.stride;
      const Tin* win_k = reinterpret_cast<const Tin*>(blk + p.so.win_k);
      const Tin* win_v = reinterpret_cast<const Tin*>(blk + p.so.win_v);
      const float* far = reinterpret_cast<const float*>(blk + p.so.far);
      const int g = (h0 + hh) / G;
      const Tin* qh = static_cast<const Tin*>(p.q) + (io * p.nq + h0 + hh) * D + part_l * DL;
      const Tin* kt = static_cast<const Tin*>(p.k) + (io * nkv + g) * D;
      const Tin* vt = static_cast<const Tin*>(p.v) + (io * nkv + g) * D;
      const long long j0 = t - K + 1 > 0 ? t - K + 1 : 0;
      const int nwin = static_cast<int>(t - j0 + 1);
      const int slot0 = static_cast<int>(j0 % K), eslot = static_cast<int>(t % K);
      auto wrow = [&](const Tin* w, const Tin* cur, int a) -> const Tin* {
        if (a == nwin - 1) return cur;
        int s2 = slot0 + a;
        if (s2 >= K) s2 -= K;
        return w + (static_cast<size_t>(s2) * nkv + g) * D;
      };
      float m = -INFINITY, den = 0.f, o[EPL];
#pragma unroll
      for (int e = 0; e < EPL; ++e) o[e] = 0.f;
      // A window of one chunk (k <= 16): its value rows are loaded together
      // with the key rows, one round trip instead of two.
      constexpr int kPre = KPC <= 16 ? KPC : 1;
      float vpre[kPre][EPL];
      if (KPC <= 16 && nwin <= KPC) {
#pragma unroll
        for (int u = 0; u < kPre; ++u)
          VecLoad<Tin, EPL>::run(wrow(win_v, vt, min(u, nwin - 1)) + lane * EPL, vpre[u]);
      }
      for (int base = 0; base < nwin; base += KPC) {
        const int cnt = min(KPC, nwin - base);
        float s;
        {  // rows past cnt are clamped to the chunk's last one (weight zero)
          const Tin* kp = wrow(win_k, kt, base + min(key, cnt - 1)) + part_l * DL;
          float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
          for (int i = 0; i < DL; i += VE) {
            float kv[VE], qv[VE];
            Load16<Tin>::run(kp + i, kv);
            Load16<Tin>::run(qh + i, qv);
#pragma unroll
            for (int e = 0; e < VE; ++e) acc[e & 3] = fmaf(qv[e], kv[e], acc[e & 3]);
          }
          s = (acc[0] + acc[1]) + (acc[2] + acc[3]);
        }
#pragma unroll
        for (int off = 1; off < LPK; off <<= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
        s = (key < cnt) ? s * p.score_scale : -INFINITY;
        const float mn = fmaxf(m, warp_max_redux(s));
        const float corr = expf(m - mn);
        const float pj = (key < cnt) ? expf(s - mn) : 0.f;
        float ps = pj;
#pragma unroll
        for (int off = 16; off >= LPK; off >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
        den = fmaf(den, corr, ps);
#pragma unroll
        for (int e = 0; e < EPL; ++e) o[e] *= corr;
        if (KPC <= 16 && nwin <= KPC) {
#pragma unroll
          for (int u = 0; u < kPre; ++u) {
            const float pc = __shfl_sync(0xffffffffu, pj, (u * LPK) & 31);  // 0 past cnt
#pragma unroll
            for (int e = 0; e < EPL; ++e) o[e] = fmaf(pc, vpre[u][e], o[e]);
          }
        } else
        for (int c0 = 0; c0 < cnt; c0 += 8) {
          float vv[8][EPL];
#pragma unroll
          for (int u = 0; u < 8; ++u)
            VecLoad<Tin, EPL>::run(wrow(win_v, vt, base + min(c0 + u, cnt - 1)) + lane * EPL, vv[u]);
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const float pc = __shfl_sync(0xffffffffu, pj, ((c0 + u) * LPK) & 31);  // 0 past cnt
#pragma unroll
            for (int e = 0; e < EPL; ++e) o[e] = fmaf(pc, vv[u][e], o[e]);
          }
        }
        m = mn;
      }
      const float inv = 1.f / den;
      float ev[EPL];
      const bool evict = t >= K;
      if (evict) VecLoad<Tin, EPL>::run(win_k + (static_cast<size_t>(eslot) * nkv + g) * D + lane * EPL, ev);
#pragma unroll
      for (int e = 0; e < EPL; ++e) {
        const float s_old = far[g * D + lane * EPL + e];
        const float s_new = evict ? ewma(p.gamma_far, s_old, ev[e]) : s_old;
        xs[r * XS + hh * D + lane * EPL + e] = fmaf(p.alpha_far, s_new, o[e] * inv);
      }
    }
  };
  if (K <= 16) near_pairs(std::integral_constant<int, 16>{});
  else near_pairs(std::integral_constant<int, 32>{});
  __syncthreads();

  // ---- (3) pool scores on the tensor cores [P3 §2.1 channel 3] -----------
  const uint32_t idesc_s = umma_idesc_bf16(kBlk, kSlots, false);
  const uint32_t idesc_c = umma_idesc_bf16(kBlk, kCW, true);
  unsigned char* xhi = xw;
  unsigned char* xlo = xw + kBlkBytes;
  for (int c = 0; c < nch; ++c) {
    if (c >= 1)  // the MMAs of chunk c-1 have finished reading the x block
      if (!mbar_wait_bounded(bar_ms, (c - 1) & 1, kMbarPollLimit, p.err)) s_bad = 1;
    stage_split_block(xs + c * kBlk, XS, xhi, xlo, tid, NT);
    fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0) {
      if (c == 0 && !mbar_wait_bounded(bar_sl, 0, kMbarPollLimit, p.err)) s_bad = 1;
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
      umma_commit(bar_ms);
    }
  }
  if (tid == 0) umma_commit(bar_sd);
  for (int r = warp; r < TB; r += NW) {  // |x|^2 per sequence while the MMAs finish
    float ss = 0.f;
    for (int e = lane; e < HS; e += 32) ss = fmaf(xs[r * XS + e], xs[r * XS + e], ss);
    ss = warp_sum(ss);
    if (lane == 0) part[r * kPartStride + kSlots] = ss;
  }
  if (!mbar_wait_bounded(bar_sd, 0, kMbarPollLimit, p.err)) s_bad = 1;
  tc_fence_after();
  {  // accumulator row r sits in lane (r % 16) + 32 (r / 16) for M = 64
    const int sp = warp & 3, colh = (warp >> 2) * 32;
    float v[32];
    tmem_ld32(tmem + (static_cast<uint32_t>(32 * sp) << 16) + colh, v);
    if (lane < 16) {
      const int r = 16 * sp + lane;
#pragma unroll
      for (int j = 0; j < 32; ++j) part[r * kPartStride + colh + j] = v[j];
    }
  }
  tc_fence_before();

  // ---- (4) cluster reduce-scatter of the pool sums, softmax(cos/T) -------
  cluster.sync();
  {
    const float* nrm = p.slot_norm + static_cast<size_t>(l) * kSlots;
    const float n0 = nrm[lane], n1 = nrm[lane + 32];
    for (int r = rank + p.CS * warp; r < TB; r += p.CS * NW) {
      float v0[kMaxCluster], v1[kMaxCluster], vs[kMaxCluster];
#pragma unroll
      for (int q = 0; q < kMaxCluster; ++q) {
        const bool in = q < p.CS;
        const float* rp = cluster.map_shared_rank(part, in ? q : 0) + r * kPartStride;
        v0[q] = in ? rp[lane] : 0.f;
        v1[q] = in ? rp[lane + 32] : 0.f;
        vs[q] = in ? rp[kSlots] : 0.f;
      }
      float d0 = 0.f, d1 = 0.f, ss = 0.f;
#pragma unroll
      for (int q = 0; q < kMaxCluster; ++q) {
        d0 += v0[q];
        d1 += v1[q];
        ss += vs[q];
      }
      const float nx = fmaxf(sqrtf(ss), kNormFloor);
      const float c0 = d0 / (nx * n0) * p.inv_temp;
      const float c1 = d1 / (nx * n1) * p.inv_temp;
      const float mx = warp_max_redux(fmaxf(c0, c1));
      const float e0 = expf(c0 - mx), e1 = expf(c1 - mx);
      const float inv = 1.f / warp_sum(e0 + e1);
      __nv_bfloat16 hb0, lb0, hb1, lb1;
      split_bf16(e0 * inv, hb0, lb0);
      split_bf16(e1 * inv, hb1, lb1);
      const int o0 = blk_off(r, lane), o1 = blk_off(r, lane + 32);
      for (int q = 0; q < p.CS; ++q) {
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
    umma_commit(bar_mc + (c & 1));
  };
  if (tid == 0) {
    issue_sem(0);
    if (nch > 1) issue_sem(1);
  }

  // ---- (5) write-back of the KV heads this CTA owns: S with the evicted key,
  // K_t and V_t into slot t mod k (every CTA has read them: barrier above)
  const bool write_ok = !s_bad;
  if (own_lo <= g_hi && write_ok) {
    const int n_own = g_hi - own_lo + 1;
    for (int idx = tid; idx < TB * n_own * D; idx += NT) {
      const int r = idx / (n_own * D);
      const long long st = rstream[r];
      if (st < 0) continue;
      const int g = own_lo + (idx / D) % n_own, i = idx % D;
      const long long t = rpos[r];
      const long long io = static_cast<long long>(li) * p.n_seq + tb * TB + r;
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
  }
  if (rank == 0 && tid < TB && rstream[tid] >= 0 && write_ok)
    *reinterpret_cast<long long*>(p.state + kHeaderBytes + rstream[tid] * p.so.stride + p.so.pos) = rpos[tid] + 1;

  // ---- (6b) per sem chunk: ring, field, fusion, clip, output -------------
  // [P3 §2.1 channels 1-2, §2.2]; thread (row, column) elements with the
  // columns consecutive, the state values loaded before the MMA wait.
  const float a_l = p.alpha_layer[l];
  for (int c = 0; c < nch; ++c) {
    float old_r[kEpt], rs_r[kEpt], fl_r[kEpt];
#pragma unroll
    for (int u = 0; u < kEpt; ++u) {
      const int idx = u * NT + tid, r = idx / kCW, e = c * kCW + idx % kCW;
      const long long st = rstream[r];
      old_r[u] = rs_r[u] = fl_r[u] = 0.f;
      if (st >= 0) {
        const unsigned char* blk = p.state + kHeaderBytes + st * p.so.stride;
        const int gi = rank * HS + e;
        old_r[u] = reinterpret_cast<const float*>(blk + p.so.ring)[static_cast<size_t>(rpos[r] & (kRing - 1)) * p.H + gi];
        rs_r[u] = reinterpret_cast<const float*>(blk + p.so.ring_sum)[gi];
        fl_r[u] = reinterpret_cast<const float*>(blk + p.so.field)[gi];
      }
    }
    const int buf = c & 1;
    if (!mbar_wait_bounded(bar_mc + buf, (c >> 1) & 1, kMbarPollLimit, p.err)) s_bad = 1;
    tc_fence_after();
    {
      const int sp = warp & 3, colh = (warp >> 2) * 32;
      float v[32];
      tmem_ld32(tmem + (static_cast<uint32_t>(32 * sp) << 16) + kSlots + buf * kCW + colh, v);
      if (lane < 16) {
        float* dst = semc + (16 * sp + lane) * kSemStride + colh;
#pragma unroll
        for (int j = 0; j < 32; j += 4)
          *reinterpret_cast<float4*>(dst + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
      }
    }
    tc_fence_before();
    __syncthreads();
    if (tid == 0 && c + 2 < nch) issue_sem(c + 2);  // overlaps the epilogue below
#pragma unroll
    for (int u = 0; u < kEpt; ++u) {
      const int idx = u * NT + tid, r = idx / kCW, cc = idx % kCW, e = c * kCW + cc;
      const long long st = rstream[r];
      if (st < 0 || !write_ok) continue;
      unsigned char* blk = p.state + kHeaderBytes + st * p.so.stride;
      const int gi = rank * HS + e;
      const float x = xs[r * XS + e];
      const float rv = (rs_r[u] - old_r[u]) + x;   // ring sum after storing x_t
      const float fv = ewma(p.ema_gamma, fl_r[u], x);  // EMA field
      float uu = rv * (1.0f / kRing) + 0.5f * fv + 0.5f * semc[r * kSemStride + cc];
      uu = fminf(fmaxf(uu, -p.clip_eps), p.clip_eps);
      reinterpret_cast<float*>(blk + p.so.ring)[static_cast<size_t>(rpos[r] & (kRing - 1)) * p.H + gi] = x;
      reinterpret_cast<float*>(blk + p.so.ring_sum)[gi] = rv;
      reinterpret_cast<float*>(blk + p.so.field)[gi] = fv;
      const long long io = static_cast<long long>(li) * p.n_seq + tb * TB + r;
      p.out[io * p.H + gi] = fmaf(a_l, uu, x);
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

template <typename Tin, int D>
cudaError_t launch_t(const DecodeParams& p, cudaStream_t s) {
  const int tiles = p.Lc * ((p.n_seq + TB - 1) / TB);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(tiles * p.CS), 1, 1);
  cfg.blockDim = dim3(NT, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(p.tile_smem);
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
  return cudaLaunchKernelEx(&cfg, decode_tile_kernel<Tin, D>, p);
}

template <typename Tin, int D>
int max_clusters_t(int cs, size_t smem) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(cs * 16), 1, 1);
  cfg.blockDim = dim3(NT, 1, 1);
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

// Dynamic shared memory of a batch-tiled decode CTA: the plan, raised to
// more than a third of the SM's shared memory so that at most two CTAs
// share an SM and their tensor-memory allocations (256 columns each) fit.
size_t decode_tile_smem_bytes(int HPC, int head_dim, size_t limit) {
  const size_t need = static_cast<size_t>(tile_plan(HPC * head_dim).total);
  return std::max(need, (limit + 1024) / 3 + 1);
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
