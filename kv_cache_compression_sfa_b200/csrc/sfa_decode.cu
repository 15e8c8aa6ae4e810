// sfa_decode.cu — fused SFA decode step: one token per (layer, sequence)
// stream, every state update in place, one launch for all layers and
// sequences.
//
// Sources (web pages):
//   [P1] "Signal Field Attention (SFA)：8KB代码实现4.16倍推理加速与248倍内存压缩"
//        §2.1 eqs. O_near, S_t, O; §2.2 O(k·d) window state.
//   [P3] "Dalin Soma SFA基于信号场注意力机制的神经网络推理加速框架"
//        §2.1 channels 1–3, §2.2 fusion, clip and alpha_layer, §2.4 ring mean.
//
// Decomposition.  A thread-block cluster of CS CTAs serves one stream; CTA
// `rank` owns query heads [rank*HPC, (rank+1)*HPC), i.e. the hidden slice
// [rank*HS, (rank+1)*HS) with HS = HPC*head_dim.  The semantic pool needs
// |x| and x·slot_j over the whole hidden vector, so each CTA forms partial
// sums over its slice and pushes them into every peer's shared memory with
// asynchronous stores that complete bytes on the peer's mbarrier; no
// cluster-wide barrier sits on the critical path.  Every CTA then adds the
// same partials in rank order, holds the same 64 softmax weights and mixes
// the slots for its own slice.
//
// Latency.  A decode step of a small batch is bound by memory latency, not
// bandwidth.  Every operand a CTA needs is brought into shared memory by the
// bulk-copy engine in a few large copies: before the kernel waits on its
// predecessor (programmatic dependent launch), the slot slice (constant;
// stored per CTA with padded rows at init), and this call's q, K_t and V_t
// too when the caller has declared them complete before the call; right
// after, the inputs otherwise, then S, field, ring sum and the window (all
// KV heads of every slot in one copy each for K and V where it fits).  Only the ring slot t mod 16 depends on the
// position and follows one round trip later, overlapped with the near field.
// All arithmetic then runs from shared memory.  A window too large for the
// shared-memory budget is read from global memory instead.
//
// Ordering.  The window slot t mod k and the far state S are read by every
// CTA that needs that KV head and written by one owner CTA (the one holding
// the group's first query head) once the partials of all ranks have reached
// it: a rank sends only after its own reads are done.  Ring, ring-sum and
// field elements belong to exactly one CTA.  The stream position is
// advanced by rank 0 at the same point.  A CTA leaves only after all peers
// have stored into it, and it never reads a peer's shared memory.
#include <cooperative_groups.h>
#include <cuda_bf16.h>

#include <type_traits>

#include "sfa_common.cuh"

namespace cg = cooperative_groups;

namespace sfa {
namespace {

constexpr int NW = kDecodeThreads / 32;
constexpr int kRedStride = kSlots + 4;            // pool partials: 64 dots, |x|^2, 3 pad
constexpr int kRedChunks = kRedStride / 4;        // float4 chunks sent to each peer
constexpr unsigned kRedBytes = kRedStride * 4u;   // bytes each CTA sends each peer
constexpr int kColsPerPass = kDecodeThreads / 2;     // epilogue: two threads per column
constexpr int kMaxCols = kMaxSlice / kColsPerPass;   // columns per thread pair
constexpr int kMaxHeadsCta = kMaxSlice / 64;         // query heads one CTA can own

// Shared-memory plan (byte offsets).  Slot rows and window slots are padded
// by 16 bytes so that lanes reading different rows at the same column hit
// distinct banks.
struct DecodePlan {
  int bars, sl, xs, red, inbox, wts, pb, mrg, qraw, kc, vc, sg, fld, rsm, wk, wv, total;
  int rec;         // bytes per staged window slot
  bool stage_win;  // window staged in shared memory
  bool whole;      // all KV heads of each slot staged (one copy each for K and V)
};

__host__ __device__ inline int a16(long long x) { return static_cast<int>((x + 15) & ~15LL); }

__host__ __device__ inline DecodePlan decode_plan(int HPC, int D, int esz, int NGm, int nkv, int K,
                                                  int budget) {
  const int HS = HPC * D;
  DecodePlan p;
  int o = 0;
  p.bars = o;  o += 32;
  p.sl = o;    o += a16(4LL * kSlots * (HS + 4));
  p.xs = o;    o += a16(4LL * HS);
  p.red = o;   o += a16(4LL * NW * kRedStride);
  p.inbox = o; o += a16(4LL * kMaxCluster * kRedStride);
  p.wts = o;   o += a16(4LL * NW * kSlots);
  p.pb = o;    o += a16(4LL * NW * 32);
  p.mrg = o;   o += a16(4LL * (NW > kMaxHeadsCta ? NW : kMaxHeadsCta) * (D + 4));
  p.qraw = o;  o += a16(static_cast<long long>(HS) * esz);
  p.kc = o;    o += a16(static_cast<long long>(NGm) * D * esz);
  p.vc = o;    o += a16(static_cast<long long>(NGm) * D * esz);
  p.sg = o;    o += a16(4LL * NGm * D);
  p.fld = o;   o += a16(4LL * HS);
  p.rsm = o;   o += a16(4LL * HS);
  // The whole window [k][n_kv][d] in one copy each for K and V where it
  // fits (few large copies instead of one per slot), else this CTA's heads
  // of each slot with 16 bytes of padding per slot, else global memory.
  p.whole = (o + 2LL * K * nkv * D * esz) <= budget;
  p.rec = p.whole ? nkv * D * esz : NGm * D * esz + 16;
  const long long win = 2LL * K * p.rec;
  p.stage_win = (o + win) <= budget;
  p.wk = o;
  p.wv = o + (p.stage_win ? K * p.rec : 0);
  if (p.stage_win) o += static_cast<int>(win);
  p.total = o;
  return p;
}

// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ unsigned map_rank(unsigned smem_addr, unsigned rank) {
  unsigned r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr), "r"(rank));
  return r;
}

// 16-byte store into a peer CTA's shared memory whose arrival is counted in
// bytes on the peer's mbarrier.
__device__ __forceinline__ void st_async_v4(unsigned addr, float4 v, unsigned bar) {
  asm volatile(
      "st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.f32 [%0], {%1, %2, %3, %4}, [%5];" ::
          "r"(addr), "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w), "r"(bar)
      : "memory");
}

// Near-field variants, chosen on the host per launch so that each kernel
// holds one copy of the near-field loop: window staged in shared memory or
// read from global memory, and window positions a warp scores at a time.
constexpr int kVarT4 = 0, kVarT8 = 1, kVarT16 = 2, kVarT32 = 3, kVarF8 = 4, kVarF32 = 5;

template <typename Tin, int D, int VAR>
__global__ void __launch_bounds__(kDecodeThreads, 2)
decode_kernel(const DecodeParams p) {
  constexpr int EPL = D / 32;  // elements of a head row per lane in P·V
  constexpr int ESZ = static_cast<int>(sizeof(Tin));
  constexpr int VE = Load16<Tin>::N;
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = static_cast<int>(cluster.block_rank());
  const int bi = blockIdx.y, li = blockIdx.z;  // call-relative sequence and layer
  const int l = p.l0 + li;                      // layer of the state
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int HPC = p.HPC, HS = HPC * D;
  const int K = p.K, G = p.G, nkv = p.nkv;
  const int h0 = rank * HPC;
  const int g_lo = h0 / G, g_hi = (h0 + HPC - 1) / G, NG = g_hi - g_lo + 1;
  const int own_lo = (h0 + G - 1) / G;

  extern __shared__ __align__(16) unsigned char smb[];
  const DecodePlan pl = decode_plan(HPC, D, ESZ, p.NGm, nkv, K, p.smem_budget);
  const int wb = pl.whole ? g_lo : 0;  // head offset of this CTA's KV heads in a staged slot
  uint64_t* bar_sl = reinterpret_cast<uint64_t*>(smb + pl.bars);
  uint64_t* bar_in = bar_sl + 1;
  uint64_t* bar_red = bar_sl + 2;
  uint64_t* bar_q = bar_sl + 3;     // this call's q, K_t, V_t
  float* sl = reinterpret_cast<float*>(smb + pl.sl);        // [64][HS+4] slot slice
  float* xs = reinterpret_cast<float*>(smb + pl.xs);        // [HS] x_t
  float* red = reinterpret_cast<float*>(smb + pl.red);      // [NW][68] per-warp pool partials
  float* inbox = reinterpret_cast<float*>(smb + pl.inbox);  // [CS][68] partials of every rank
  float* wts = reinterpret_cast<float*>(smb + pl.wts) + warp * kSlots;  // this warp's weights
  float* pb = reinterpret_cast<float*>(smb + pl.pb) + warp * 32;        // this warp's chunk weights
  float* mrg = reinterpret_cast<float*>(smb + pl.mrg);     // [head][key part][D + 4] partial softmax
  Tin* qraw = reinterpret_cast<Tin*>(smb + pl.qraw);        // [HS] queries as stored
  Tin* kc = reinterpret_cast<Tin*>(smb + pl.kc);            // [NG][D] K_t
  Tin* vc = reinterpret_cast<Tin*>(smb + pl.vc);            // [NG][D] V_t
  float* sg = reinterpret_cast<float*>(smb + pl.sg);        // [NG][D] S before this step
  float* fld = reinterpret_cast<float*>(smb + pl.fld);      // [HS] field before this step
  float* rsm = reinterpret_cast<float*>(smb + pl.rsm);      // [HS] ring sum before this step
  unsigned char* wk = smb + pl.wk;                          // [K][rec] window keys
  unsigned char* wv = smb + pl.wv;                          // [K][rec] window values
  __shared__ long long s_pos;
  __shared__ int s_ok;

  if (tid == 0) {
    mbar_init(bar_sl, 1);
    mbar_init(bar_in, 1);
    mbar_init(bar_red, 1);
    mbar_init(bar_q, 1);
    mbar_fence_init();
    // the partials of all CS ranks (this one included) complete the phase
    mbar_arrive_expect_tx(bar_red, static_cast<unsigned>(p.CS) * kRedBytes);
  }
  __syncthreads();
  // Barrier initialisation visible to the peers before any of them stores
  // into this CTA (they wait on this arrival just before sending).
  cluster_arrive();
  pdl_trigger();

  // Slot slice: constant since sfa_init, so it may be fetched before the
  // previous kernel of the stream has finished.
  // One copy: the slice is stored contiguously with padded rows at init.
  if (tid == 0) {
    const unsigned bytes = static_cast<unsigned>(kSlots * (HS + 4) * 4);
    mbar_arrive_expect_tx(bar_sl, bytes);
    bulk_g2s(sl, p.slot_dec + (static_cast<size_t>(l) * p.CS + rank) * kSlots * (HS + 4), bytes, bar_sl);
  }
  // Other per-layer constants: slot norms (lane j: slots j, j+32; every
  // warp forms the softmax itself) and alpha_layer.
  const float* nrm = p.slot_norm + static_cast<size_t>(l) * kSlots;
  const float inrm0 = 1.f / nrm[lane], inrm1 = 1.f / nrm[lane + 32];
  const float a_l = p.alpha_layer[l];

  // This call's query slice and K_t, V_t of the CTA's KV heads.  A kernel
  // still running on the stream may be writing them, so by default they are
  // fetched after the wait below.  When the caller has declared them
  // complete before the call (sfa_set_decode_input_prefetch), they are
  // fetched before it: decode inputs usually come from HBM, and that takes
  // their latency off the critical path.
  const long long io = static_cast<long long>(li) * p.n_seq + bi;  // input / output row
  const Tin* qin = static_cast<const Tin*>(p.q) + (io * p.nq + h0) * D;
  const Tin* kin = static_cast<const Tin*>(p.k) + io * nkv * D;
  const Tin* vin = static_cast<const Tin*>(p.v) + io * nkv * D;
  auto fetch_inputs = [&]() {
    if (tid == 32) {
      const unsigned hb = static_cast<unsigned>(NG * D * ESZ);
      mbar_arrive_expect_tx(bar_q, static_cast<unsigned>(HS * ESZ) + 2u * hb);
      bulk_g2s(qraw, qin, static_cast<unsigned>(HS * ESZ), bar_q);
      bulk_g2s(kc, kin + g_lo * D, hb, bar_q);
      bulk_g2s(vc, vin + g_lo * D, hb, bar_q);
    }
  };
  if (p.inputs_early) fetch_inputs();

  pdl_wait();  // the state (and, by default, the inputs) may be written by the previous kernel
  if (!p.inputs_early) fetch_inputs();

  // Sequence served: from the caller's list, checked against the batch (an
  // index out of range leaves the cluster without touching the state).
  int b = bi;
  if (p.seq_ids) b = __ldcg(p.seq_ids + bi);
  const bool b_ok = b >= 0 && b < p.B;
  if (!b_ok) b = 0;
  const long long stream = static_cast<long long>(l) * p.B + b;  // state stream
  unsigned char* blk = p.state + kHeaderBytes + stream * p.so.stride;
  Tin* win_k = reinterpret_cast<Tin*>(blk + p.so.win_k);
  Tin* win_v = reinterpret_cast<Tin*>(blk + p.so.win_v);
  float* far = reinterpret_cast<float*>(blk + p.so.far);
  float* field = reinterpret_cast<float*>(blk + p.so.field);
  float* ring_sum = reinterpret_cast<float*>(blk + p.so.ring_sum);
  float* ring = reinterpret_cast<float*>(blk + p.so.ring);

  if (tid == 0) {  // header and position: independent loads, one round trip
    const uint4 h0v = __ldcg(reinterpret_cast<const uint4*>(p.state));
    const uint4 h1v = __ldcg(reinterpret_cast<const uint4*>(p.state + 16));
    const long long pos = __ldcg(reinterpret_cast<const long long*>(blk + p.so.pos));
    StateHeader hd;
    reinterpret_cast<uint4*>(&hd)[0] = h0v;
    reinterpret_cast<uint4*>(&hd)[1] = h1v;
    s_ok = (hd.magic == kMagic) & (hd.cfg_hash == p.cfg_hash) & (hd.batch == p.B) &
           (hd.n_layers == p.L);
    s_pos = pos;
  }
  if (warp == 1) {  // the rest of this stream's state, one batch of copies
    const unsigned hb = static_cast<unsigned>(NG * D * ESZ);
    unsigned bytes = static_cast<unsigned>(NG * D * 4) + 2u * static_cast<unsigned>(HS * 4);
    if (pl.stage_win) bytes += 2u * static_cast<unsigned>(K) * (pl.whole ? static_cast<unsigned>(pl.rec) : hb);
    if (lane == 0) mbar_arrive_expect_tx(bar_in, bytes);
    __syncwarp();
    if (lane == 3) bulk_g2s(sg, far + g_lo * D, static_cast<unsigned>(NG * D * 4), bar_in);
    if (lane == 4) bulk_g2s(fld, field + rank * HS, static_cast<unsigned>(HS * 4), bar_in);
    if (lane == 5) bulk_g2s(rsm, ring_sum + rank * HS, static_cast<unsigned>(HS * 4), bar_in);
    if (pl.whole) {
      if (lane == 6) bulk_g2s(wk, win_k, static_cast<unsigned>(K * pl.rec), bar_in);
      if (lane == 7) bulk_g2s(wv, win_v, static_cast<unsigned>(K * pl.rec), bar_in);
    } else if (pl.stage_win)
      for (int s = lane; s < K; s += 32) {
        const size_t off = (static_cast<size_t>(s) * nkv + g_lo) * D;
        bulk_g2s(wk + s * pl.rec, win_k + off, hb, bar_in);
        bulk_g2s(wv + s * pl.rec, win_v + off, hb, bar_in);
      }
  }
  __syncthreads();
  if (!s_ok || !b_ok) {  // uniform over the cluster (same header, same sequence)
    mbar_wait_bounded(bar_sl, 0, kMbarPollLimit, p.err);  // no copy may land after exit
    mbar_wait_bounded(bar_q, 0, kMbarPollLimit, p.err);
    mbar_wait_bounded(bar_in, 0, kMbarPollLimit, p.err);
    cluster_wait();
    if (tid == 0 && rank == 0) {
      if (!s_ok && bi == 0 && li == 0) latch_error(p.err, SFA_ERR_STATE_MISMATCH);
      if (s_ok && !b_ok) latch_error(p.err, SFA_ERR_INVALID_ARG);
    }
    return;
  }
  const long long t = s_pos;
  const long long j0 = (t - K + 1 > 0) ? t - K + 1 : 0;
  const int nwin = static_cast<int>(t - j0 + 1);
  const int eslot = static_cast<int>(t % K);   // slot of t (and of the evicted t-k)
  const int slot0 = static_cast<int>(j0 % K);  // slot of the first window position
  const bool evict = t >= K;
  const int rslot = static_cast<int>(t % kRing);

  // Epilogue mapping: lanes l and l+16 of warp w share slice column
  // 16w + (l & 15) (+ 128 m), each mixing half of the slots.  The ring slot
  // being replaced depends on t: one round trip later, overlapped with the
  // near field.
  const int ecol = warp * 16 + (lane & 15), ehalf = lane >> 4;
  const int ncol = (HS - ecol + kColsPerPass - 1) / kColsPerPass;  // uniform over a warp
  float ring_old[kMaxCols];
  float* ring_row = ring + static_cast<size_t>(rslot) * p.H + rank * HS;
#pragma unroll
  for (int m = 0; m < kMaxCols; ++m)
    ring_old[m] = (m < ncol && ehalf == 0) ? ring_row[ecol + m * kColsPerPass] : 0.f;

  bool ok = mbar_wait_bounded(bar_in, 0, kMbarPollLimit, p.err);
  ok = mbar_wait_bounded(bar_q, 0, kMbarPollLimit, p.err) && ok;

  // Window slot of the a-th window position (a = 0 .. nwin-1 is position
  // j0+a).
  auto wslot = [&](int a) -> int {
    const int s2 = slot0 + a;
    return s2 >= K ? s2 - K : s2;
  };

  // (1)-(2) near field per query head [P1 §2.1 eq. O_near].  WPH warps share
  // a head, each taking a contiguous part of the window; a warp scores KPC
  // positions at a time with LPK = 32/KPC lanes per position splitting the
  // q·K dot product, keeps an online softmax (max m, denominator, P·V with
  // lanes over head dims) and leaves it in `mrg` for the merge below.
  // STAGED: window rows in shared memory (else read from global memory).
  int wph = 1;
  while (wph * 2 * HPC <= NW) wph *= 2;
  const int gw = warp / wph, sw = warp % wph, n_gw = NW / wph;
  const int per = (nwin + wph - 1) / wph;
  const int k_lo = min(nwin, sw * per), k_hi = min(nwin, k_lo + per);
  auto near_part = [&](auto staged_c, auto kpc_c) {
    constexpr bool STAGED = decltype(staged_c)::value;
    constexpr int KPC = decltype(kpc_c)::value;
    constexpr int LPK = 32 / KPC;
    constexpr int DL = D / LPK;  // dims of the score per lane
    auto krow = [&](int a, int gg) -> const Tin* {
      if (a == nwin - 1) return kc + gg * D;
      const int s2 = wslot(a);
      if constexpr (STAGED) return reinterpret_cast<const Tin*>(wk + s2 * pl.rec) + (wb + gg) * D;
      else return win_k + (static_cast<size_t>(s2) * nkv + g_lo + gg) * D;
    };
    auto vrow = [&](int a, int gg) -> const Tin* {
      if (a == nwin - 1) return vc + gg * D;
      const int s2 = wslot(a);
      if constexpr (STAGED) return reinterpret_cast<const Tin*>(wv + s2 * pl.rec) + (wb + gg) * D;
      else return win_v + (static_cast<size_t>(s2) * nkv + g_lo + gg) * D;
    };
    const int key = lane / LPK, part = lane % LPK;
    for (int hh = gw; hh < HPC; hh += n_gw) {
      const int gg = (h0 + hh) / G - g_lo;
      const Tin* qh = qraw + hh * D + part * DL;
      float m = -INFINITY, den = 0.f, o[EPL];
#pragma unroll
      for (int e = 0; e < EPL; ++e) o[e] = 0.f;
      for (int base = k_lo; base < k_hi; base += KPC) {
        const int cnt = min(KPC, k_hi - base);
        // Rows past cnt are clamped to the chunk's last one (their weight
        // is zero), so every load is unconditional and issued at once.
        float s;
        {
          const Tin* kp = krow(base + min(key, cnt - 1), gg) + part * DL;
          float acc[4] = {0.f, 0.f, 0.f, 0.f};  // independent chains
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
        if (part == 0) pb[key] = pj;  // weights of the chunk, read back as broadcasts
        __syncwarp();
#pragma unroll
        for (int e = 0; e < EPL; ++e) o[e] *= corr;
        for (int c0 = 0; c0 < cnt; c0 += 4) {
          float vv[4][EPL];
#pragma unroll
          for (int u = 0; u < 4; ++u)
            VecLoad<Tin, EPL>::run(vrow(base + min(c0 + u, cnt - 1), gg) + lane * EPL, vv[u]);
          const float4 pc = *reinterpret_cast<const float4*>(pb + c0);  // 0 past cnt
#pragma unroll
          for (int e = 0; e < EPL; ++e)
            o[e] = fmaf(pc.x, vv[0][e], fmaf(pc.y, vv[1][e], fmaf(pc.z, vv[2][e], fmaf(pc.w, vv[3][e], o[e]))));
        }
        __syncwarp();  // pb is rewritten by the next chunk
        m = mn;
      }
      float* mp = mrg + (hh * wph + sw) * (D + 4);
#pragma unroll
      for (int e = 0; e < EPL; ++e) mp[lane * EPL + e] = o[e];
      if (lane == 0) {
        mp[D] = m;
        mp[D + 1] = den;
      }
    }
  };
  {
    constexpr bool kStaged = VAR < kVarF8;
    constexpr int kKpc = (VAR == kVarT4) ? 4 : (VAR == kVarT8 || VAR == kVarF8) ? 8 : (VAR == kVarT16) ? 16 : 32;
    near_part(std::integral_constant<bool, kStaged>{}, std::integral_constant<int, kKpc>{});
  }
  __syncthreads();

  // (3)-(4) merge the parts of each head (log-sum-exp), far field with the
  // evicted key [P1 §2.1 eq. S_t], x = O_near + alpha_far * S [P1 §2.1 eq. O].
  for (int idx = tid; idx < HS; idx += kDecodeThreads) {
    const int hh = idx / D, i = idx % D;
    const float* mp = mrg + hh * wph * (D + 4);
    float mstar = -INFINITY;
    for (int q = 0; q < wph; ++q) mstar = fmaxf(mstar, mp[q * (D + 4) + D]);
    float num = 0.f, den = 0.f;
    for (int q = 0; q < wph; ++q) {
      const float sc = expf(mp[q * (D + 4) + D] - mstar);
      num = fmaf(sc, mp[q * (D + 4) + i], num);
      den = fmaf(sc, mp[q * (D + 4) + D + 1], den);
    }
    const int gg = (h0 + hh) / G - g_lo;
    float s_new = sg[gg * D + i];
    if (evict) {
      const Tin* er = pl.stage_win ? reinterpret_cast<const Tin*>(wk + eslot * pl.rec) + (wb + gg) * D
                                   : win_k + (static_cast<size_t>(eslot) * nkv + g_lo + gg) * D;
      s_new = ewma(p.gamma_far, s_new, to_f32<Tin>(er[i]));
    }
    xs[idx] = fmaf(p.alpha_far, s_new, num / den);
  }
  __syncthreads();

  // (7a) pool partial sums over this slice [P3 §2.1 channel 3]: warp w takes
  // an eighth of the slice, lane j slots j and j+32.
  ok = mbar_wait_bounded(bar_sl, 0, kMbarPollLimit, p.err) && ok;
  {
    const int q4 = HS / NW;  // elements per warp
    const float* x0 = xs + warp * q4;
    const float* r0 = sl + lane * (HS + 4) + warp * q4;
    const float* r1 = sl + (lane + 32) * (HS + 4) + warp * q4;
    float4 a0 = make_float4(0.f, 0.f, 0.f, 0.f), a1 = a0;  // one chain per component
    float ss = 0.f;
#pragma unroll 4
    for (int e = 0; e < q4; e += 4) {
      const float4 xv = *reinterpret_cast<const float4*>(x0 + e);
      const float4 a = *reinterpret_cast<const float4*>(r0 + e);
      const float4 c = *reinterpret_cast<const float4*>(r1 + e);
      a0.x = fmaf(xv.x, a.x, a0.x); a0.y = fmaf(xv.y, a.y, a0.y);
      a0.z = fmaf(xv.z, a.z, a0.z); a0.w = fmaf(xv.w, a.w, a0.w);
      a1.x = fmaf(xv.x, c.x, a1.x); a1.y = fmaf(xv.y, c.y, a1.y);
      a1.z = fmaf(xv.z, c.z, a1.z); a1.w = fmaf(xv.w, c.w, a1.w);
    }
    for (int e = lane; e < q4; e += 32) ss = fmaf(x0[e], x0[e], ss);
    ss = warp_sum(ss);
    red[warp * kRedStride + lane] = (a0.x + a0.y) + (a0.z + a0.w);
    red[warp * kRedStride + lane + 32] = (a1.x + a1.y) + (a1.z + a1.w);
    if (lane < kRedStride - kSlots) red[warp * kRedStride + kSlots + lane] = (lane == 0) ? ss : 0.f;
  }
  __syncthreads();
  // Every peer has initialised its barriers (arrival at the top).
  cluster_wait();

  // (7b) push this CTA's partials (sum over its warps) to every rank's inbox
  // row `rank`; the stores complete bytes on the receiver's barrier.
  for (int idx = tid; idx < p.CS * kRedChunks; idx += kDecodeThreads) {
    const int peer = idx / kRedChunks, c = idx % kRedChunks;
    float4 v = *reinterpret_cast<const float4*>(red + c * 4);
#pragma unroll
    for (int w = 1; w < NW; ++w) {
      const float4 u = *reinterpret_cast<const float4*>(red + w * kRedStride + c * 4);
      v.x += u.x; v.y += u.y; v.z += u.z; v.w += u.w;
    }
    st_async_v4(map_rank(smem_u32(inbox + rank * kRedStride + c * 4), peer), v,
                map_rank(smem_u32(bar_red), peer));
  }
  // All ranks' partials have landed here; every rank has also finished
  // reading the window slot, S and position of this stream.
  ok = mbar_wait_bounded(bar_red, 0, kMbarPollLimit, p.err) && ok;

  // Sum in rank order (identical in every CTA and warp), softmax(cos/T);
  // each warp keeps its own copy of the weights.
  {
    float v0[kMaxCluster], v1[kMaxCluster], vs[kMaxCluster];
#pragma unroll
    for (int r = 0; r < kMaxCluster; ++r) {
      const bool in = r < p.CS;
      v0[r] = in ? inbox[r * kRedStride + lane] : 0.f;
      v1[r] = in ? inbox[r * kRedStride + lane + 32] : 0.f;
      vs[r] = in ? inbox[r * kRedStride + kSlots] : 0.f;
    }
    float d0 = 0.f, d1 = 0.f, ss = 0.f;
#pragma unroll
    for (int r = 0; r < kMaxCluster; ++r) {
      d0 += v0[r];
      d1 += v1[r];
      ss += vs[r];
    }
    const float inx = p.inv_temp / fmaxf(sqrtf(ss), kNormFloor);
    const float c0 = d0 * inrm0 * inx;
    const float c1 = d1 * inrm1 * inx;
    const float mx = warp_max_redux(fmaxf(c0, c1));
    const float e0 = expf(c0 - mx), e1 = expf(c1 - mx);
    const float inv = 1.f / warp_sum(e0 + e1);
    wts[lane] = e0 * inv;
    wts[lane + 32] = e1 * inv;
    __syncwarp();
  }

  // (5)(6)(7c)(8): ring, field, semantic mix, fusion, clip, scale, output.
  // Half h of a column's thread pair mixes slots 8i + 4h .. 8i + 4h + 3
  // (rows four apart: the two halves hit disjoint banks).
  if (ok) {
#pragma unroll
    for (int m = 0; m < kMaxCols; ++m) {
      if (m >= ncol) break;
      const int c = ecol + m * kColsPerPass;
      float a[4] = {0.f, 0.f, 0.f, 0.f};  // independent chains
#pragma unroll
      for (int j8 = 0; j8 < kSlots; j8 += 8) {
        const int j = j8 + 4 * ehalf;
        const float4 w4 = *reinterpret_cast<const float4*>(wts + j);
        a[0] = fmaf(w4.x, sl[j * (HS + 4) + c], a[0]);
        a[1] = fmaf(w4.y, sl[(j + 1) * (HS + 4) + c], a[1]);
        a[2] = fmaf(w4.z, sl[(j + 2) * (HS + 4) + c], a[2]);
        a[3] = fmaf(w4.w, sl[(j + 3) * (HS + 4) + c], a[3]);
      }
      float sem = (a[0] + a[1]) + (a[2] + a[3]);
      sem += __shfl_xor_sync(0xffffffffu, sem, 16);
      if (ehalf == 0) {
        const float x = xs[c];
        const float rv = (rsm[c] - ring_old[m]) + x;   // ring sum after storing x_t
        const float fv = ewma(p.ema_gamma, fld[c], x);  // EMA field
        float u = rv * (1.0f / kRing) + 0.5f * fv + 0.5f * sem;
        u = fminf(fmaxf(u, -p.clip_eps), p.clip_eps);
        const int gi = rank * HS + c;
        ring_row[c] = x;
        ring_sum[gi] = rv;
        field[gi] = fv;
        store_result(p.out_mode, p.res, io * p.H + gi, a_l, u, x);
      }
    }
  }

  // (1)(2) write-back of the KV heads this CTA owns, from the staged copies:
  // S with the evicted key, then K_t, V_t into slot t mod k.  Every CTA of
  // the cluster has read the old values (its partials have arrived).
  if (ok) {
    const int n_own = g_hi - own_lo + 1;
    for (int idx = tid; idx < n_own * D; idx += kDecodeThreads) {
      const int gg = own_lo - g_lo + idx / D;
      const int i = idx % D;
      float s = sg[gg * D + i];
      if (evict) {
        const int s2 = eslot;
        const Tin* er = pl.stage_win ? reinterpret_cast<const Tin*>(wk + s2 * pl.rec) + (wb + gg) * D
                                     : win_k + (static_cast<size_t>(s2) * nkv + g_lo + gg) * D;
        s = ewma(p.gamma_far, s, to_f32<Tin>(er[i]));
      }
      const size_t wo = (static_cast<size_t>(eslot) * nkv + g_lo + gg) * D + i;
      far[(g_lo + gg) * D + i] = s;
      win_k[wo] = kc[gg * D + i];
      win_v[wo] = vc[gg * D + i];
    }
    if (rank == 0 && tid == 0) *reinterpret_cast<long long*>(blk + p.so.pos) = t + 1;
  }
}

// The near-field variant a launch needs (the kernel's own choice of warps
// per head and window staging, made on the host).
int decode_variant(const DecodeParams& p, const DecodePlan& pl) {
  int wph = 1;
  while (wph * 2 * p.HPC <= NW) wph *= 2;
  const int pmax = (p.K + wph - 1) / wph;  // most positions a warp ever takes
  if (pl.stage_win) return pmax <= 4 ? kVarT4 : pmax <= 8 ? kVarT8 : pmax <= 16 ? kVarT16 : kVarT32;
  return pmax <= 8 ? kVarF8 : kVarF32;
}

template <typename Tin, int D, int VAR>
cudaError_t launch_v(const DecodeParams& p, const DecodePlan& pl, cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.CS, p.n_seq, p.Lc);
  cfg.blockDim = dim3(kDecodeThreads, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(pl.total);
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
  return cudaLaunchKernelEx(&cfg, decode_kernel<Tin, D, VAR>, p);
}

template <typename Tin, int D>
cudaError_t launch_t(const DecodeParams& p, cudaStream_t s) {
  const DecodePlan pl = decode_plan(p.HPC, D, static_cast<int>(sizeof(Tin)), p.NGm, p.nkv, p.K, p.smem_budget);
  switch (decode_variant(p, pl)) {
    case kVarT4: return launch_v<Tin, D, kVarT4>(p, pl, s);
    case kVarT8: return launch_v<Tin, D, kVarT8>(p, pl, s);
    case kVarT16: return launch_v<Tin, D, kVarT16>(p, pl, s);
    case kVarT32: return launch_v<Tin, D, kVarT32>(p, pl, s);
    case kVarF8: return launch_v<Tin, D, kVarF8>(p, pl, s);
    default: return launch_v<Tin, D, kVarF32>(p, pl, s);
  }
}

template <typename Tin, int D, int VAR>
cudaError_t prepare_v(int optin) {
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, decode_kernel<Tin, D, VAR>);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(decode_kernel<Tin, D, VAR>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             optin - static_cast<int>(fa.sharedSizeBytes));
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(decode_kernel<Tin, D, VAR>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  return e;
}

template <typename Tin, int D>
cudaError_t prepare_t(int optin) {
  cudaError_t e = prepare_v<Tin, D, kVarT4>(optin);
  if (e == cudaSuccess) e = prepare_v<Tin, D, kVarT8>(optin);
  if (e == cudaSuccess) e = prepare_v<Tin, D, kVarT16>(optin);
  if (e == cudaSuccess) e = prepare_v<Tin, D, kVarT32>(optin);
  if (e == cudaSuccess) e = prepare_v<Tin, D, kVarF8>(optin);
  if (e == cudaSuccess) e = prepare_v<Tin, D, kVarF32>(optin);
  return e;
}

// Clusters of `cs` CTAs resident at once (shared memory bounds it; the
// variants differ only in the near-field loop).
template <typename Tin, int D>
int max_clusters_t(int cs, size_t smem) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(cs), 16, 1);
  cfg.blockDim = dim3(kDecodeThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cs;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, decode_kernel<Tin, D, kVarT32>, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}

}  // namespace

// Shared memory of one decode CTA; the window is staged when it fits in
// `budget` bytes together with everything else.
size_t decode_smem_bytes(int HPC, int head_dim, int esz, int NGm, int nkv, int K, int budget) {
  return static_cast<size_t>(decode_plan(HPC, head_dim, esz, NGm, nkv, K, budget).total);
}

int decode_max_active_clusters(int cs, size_t smem, int in_dtype, int head_dim) {
  if (in_dtype == SFA_F32) return head_dim == 64 ? max_clusters_t<float, 64>(cs, smem) : max_clusters_t<float, 128>(cs, smem);
  return head_dim == 64 ? max_clusters_t<__nv_bfloat16, 64>(cs, smem)
                        : max_clusters_t<__nv_bfloat16, 128>(cs, smem);
}

cudaError_t decode_prepare(int device) {
  int optin = 0;
  cudaError_t e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, device);
  if (e == cudaSuccess) e = prepare_t<float, 64>(optin);
  if (e == cudaSuccess) e = prepare_t<float, 128>(optin);
  if (e == cudaSuccess) e = prepare_t<__nv_bfloat16, 64>(optin);
  if (e == cudaSuccess) e = prepare_t<__nv_bfloat16, 128>(optin);
  return e;
}

cudaError_t launch_decode(const DecodeParams& p, int in_dtype, int head_dim, cudaStream_t s) {
  if (in_dtype == SFA_F32) {
    return head_dim == 64 ? launch_t<float, 64>(p, s) : launch_t<float, 128>(p, s);
  }
  return head_dim == 64 ? launch_t<__nv_bfloat16, 64>(p, s) : launch_t<__nv_bfloat16, 128>(p, s);
}

}  // namespace sfa
