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
// sums over its slice and the cluster adds them through distributed shared
// memory; every CTA then holds the same 64 softmax weights and mixes the
// slots for its own slice.
//
// Latency.  A decode step of a small batch is bound by memory latency, not
// bandwidth.  Every operand a CTA needs is brought into shared memory by the
// bulk-copy engine in one batch: the slot slice before the kernel waits on
// its predecessor (programmatic dependent launch; slots are constant), the
// query slice, the new key/value, the window, S, field and ring sum right
// after.  Only the ring slot t mod 16 depends on the position and follows
// one round trip later, overlapped with the near field.  All arithmetic
// then runs from shared memory.  A window too large for the shared-memory
// budget is read from global memory instead.
//
// Ordering.  The window slot t mod k and the far state S are read by every
// CTA that needs that KV head and written by one owner CTA (the one holding
// the group's first query head) after the first cluster barrier, when all
// reads are done.  Ring, ring-sum and field elements belong to exactly one
// CTA.  The stream position is advanced by rank 0 after the same barrier.
#include <cooperative_groups.h>
#include <cuda_bf16.h>

#include "sfa_common.cuh"

namespace cg = cooperative_groups;

namespace sfa {
namespace {

constexpr int NW = kDecodeThreads / 32;
constexpr int kRedStride = kSlots + 4;  // per-warp partials: 64 dots + |x|^2

// Shared-memory plan (byte offsets).  Slot rows and window slots are padded
// by 16 bytes so that lanes reading different rows at the same column hit
// distinct banks.
struct DecodePlan {
  int bars, sl, qf, xs, red, part, wts, qraw, kc, vc, sg, fld, rsm, wk, wv, total;
  int rec;         // bytes per staged window slot (NGm heads + pad)
  bool stage_win;  // window staged in shared memory
};

__host__ __device__ inline int a16(long long x) { return static_cast<int>((x + 15) & ~15LL); }

__host__ __device__ inline DecodePlan decode_plan(int HPC, int D, int esz, int NGm, int K,
                                                  int budget) {
  const int HS = HPC * D;
  DecodePlan p;
  int o = 0;
  p.bars = o;  o += 16;
  p.sl = o;    o += a16(4LL * kSlots * (HS + 4));
  p.qf = o;    o += a16(4LL * HS);
  p.xs = o;    o += a16(4LL * HS);
  p.red = o;   o += a16(4LL * NW * kRedStride);
  p.part = o;  o += a16(4LL * kRedStride);
  p.wts = o;   o += a16(4LL * kSlots);
  p.qraw = o;  o += a16(static_cast<long long>(HS) * esz);
  p.kc = o;    o += a16(static_cast<long long>(NGm) * D * esz);
  p.vc = o;    o += a16(static_cast<long long>(NGm) * D * esz);
  p.sg = o;    o += a16(4LL * NGm * D);
  p.fld = o;   o += a16(4LL * HS);
  p.rsm = o;   o += a16(4LL * HS);
  p.rec = NGm * D * esz + 16;
  const long long win = 2LL * K * p.rec;
  p.stage_win = (o + win) <= budget;
  p.wk = o;
  p.wv = o + (p.stage_win ? K * p.rec : 0);
  if (p.stage_win) o += static_cast<int>(win);
  p.total = o;
  return p;
}

template <typename Tin, int D>
__global__ void __launch_bounds__(kDecodeThreads)
decode_kernel(const DecodeParams p) {
  constexpr int EPL = D / 32;  // elements of a head row per lane
  constexpr int ESZ = static_cast<int>(sizeof(Tin));
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = static_cast<int>(cluster.block_rank());
  const int b = blockIdx.y, l = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int HPC = p.HPC, HS = HPC * D;
  const int K = p.K, G = p.G, nkv = p.nkv;
  const int h0 = rank * HPC;
  const int g_lo = h0 / G, g_hi = (h0 + HPC - 1) / G, NG = g_hi - g_lo + 1;
  const int own_lo = (h0 + G - 1) / G;

  extern __shared__ __align__(16) unsigned char smb[];
  const DecodePlan pl = decode_plan(HPC, D, ESZ, p.NGm, K, p.smem_budget);
  uint64_t* bar_sl = reinterpret_cast<uint64_t*>(smb + pl.bars);
  uint64_t* bar_in = bar_sl + 1;
  float* sl = reinterpret_cast<float*>(smb + pl.sl);      // [64][HS+4] slot slice
  float* qf = reinterpret_cast<float*>(smb + pl.qf);      // [HS] queries, fp32
  float* xs = reinterpret_cast<float*>(smb + pl.xs);      // [HS] x_t
  float* red = reinterpret_cast<float*>(smb + pl.red);    // [NW][68] per-warp pool partials
  float* part = reinterpret_cast<float*>(smb + pl.part);  // [68] CTA pool partials
  float* wts = reinterpret_cast<float*>(smb + pl.wts);    // [64] pool weights
  Tin* qraw = reinterpret_cast<Tin*>(smb + pl.qraw);      // [HS] queries as stored
  Tin* kc = reinterpret_cast<Tin*>(smb + pl.kc);          // [NG][D] K_t
  Tin* vc = reinterpret_cast<Tin*>(smb + pl.vc);          // [NG][D] V_t
  float* sg = reinterpret_cast<float*>(smb + pl.sg);      // [NG][D] S before this step
  float* fld = reinterpret_cast<float*>(smb + pl.fld);    // [HS] field before this step
  float* rsm = reinterpret_cast<float*>(smb + pl.rsm);    // [HS] ring sum before this step
  unsigned char* wk = smb + pl.wk;                        // [K][rec] window keys
  unsigned char* wv = smb + pl.wv;                        // [K][rec] window values
  __shared__ long long s_pos;
  __shared__ int s_ok;

  if (tid == 0) {
    mbar_init(bar_sl, 1);
    mbar_init(bar_in, 1);
    mbar_fence_init();
  }
  __syncthreads();
  pdl_trigger();

  // Slot slice: constant since sfa_init, so it may be fetched before the
  // previous kernel of the stream has finished.
  const float* slot_base = p.slots + static_cast<size_t>(l) * kSlots * p.H + static_cast<size_t>(rank) * HS;
  if (warp == 0) {
    if (lane == 0) mbar_arrive_expect_tx(bar_sl, kSlots * HS * 4u);
    __syncwarp();
    for (int j = lane; j < kSlots; j += 32)
      bulk_g2s(sl + j * (HS + 4), slot_base + static_cast<size_t>(j) * p.H, HS * 4u, bar_sl);
  }

  // Other per-layer constants: slot norms and alpha_layer.
  float nrm0 = 0.f, nrm1 = 0.f, a_l = 0.f;
  if (warp == 0) {
    const float* nrm = p.slot_norm + static_cast<size_t>(l) * kSlots;
    nrm0 = nrm[lane];
    nrm1 = nrm[lane + 32];
  }
  if (tid < HS / 4) a_l = p.alpha_layer[l];

  pdl_wait();  // state and inputs may be written by the previous kernel

  const long long stream = static_cast<long long>(l) * p.B + b;
  unsigned char* blk = p.state + kHeaderBytes + stream * p.so.stride;
  Tin* win_k = reinterpret_cast<Tin*>(blk + p.so.win_k);
  Tin* win_v = reinterpret_cast<Tin*>(blk + p.so.win_v);
  float* far = reinterpret_cast<float*>(blk + p.so.far);
  float* field = reinterpret_cast<float*>(blk + p.so.field);
  float* ring_sum = reinterpret_cast<float*>(blk + p.so.ring_sum);
  float* ring = reinterpret_cast<float*>(blk + p.so.ring);
  const Tin* qin = static_cast<const Tin*>(p.q) + (stream * p.nq + h0) * D;
  const Tin* kin = static_cast<const Tin*>(p.k) + stream * nkv * D;
  const Tin* vin = static_cast<const Tin*>(p.v) + stream * nkv * D;

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
  if (warp == 1) {  // everything else of this stream, one batch of copies
    const unsigned hb = static_cast<unsigned>(NG * D * ESZ);
    unsigned bytes = static_cast<unsigned>(HS * ESZ) + 2u * hb + static_cast<unsigned>(NG * D * 4) +
                     2u * static_cast<unsigned>(HS * 4);
    if (pl.stage_win) bytes += 2u * static_cast<unsigned>(K) * hb;
    if (lane == 0) mbar_arrive_expect_tx(bar_in, bytes);
    __syncwarp();
    if (lane == 0) bulk_g2s(qraw, qin, static_cast<unsigned>(HS * ESZ), bar_in);
    if (lane == 1) bulk_g2s(kc, kin + g_lo * D, hb, bar_in);
    if (lane == 2) bulk_g2s(vc, vin + g_lo * D, hb, bar_in);
    if (lane == 3) bulk_g2s(sg, far + g_lo * D, static_cast<unsigned>(NG * D * 4), bar_in);
    if (lane == 4) bulk_g2s(fld, field + rank * HS, static_cast<unsigned>(HS * 4), bar_in);
    if (lane == 5) bulk_g2s(rsm, ring_sum + rank * HS, static_cast<unsigned>(HS * 4), bar_in);
    if (pl.stage_win)
      for (int s = lane; s < K; s += 32) {
        const size_t off = (static_cast<size_t>(s) * nkv + g_lo) * D;
        bulk_g2s(wk + s * pl.rec, win_k + off, hb, bar_in);
        bulk_g2s(wv + s * pl.rec, win_v + off, hb, bar_in);
      }
  }
  __syncthreads();
  if (!s_ok) {  // the same header for every CTA: the whole grid leaves here
    mbar_wait_bounded(bar_sl, 0, kMbarPollLimit, p.err);  // no copy may land after exit
    mbar_wait_bounded(bar_in, 0, kMbarPollLimit, p.err);
    if (tid == 0 && rank == 0 && b == 0 && l == 0) latch_error(p.err, SFA_ERR_STATE_MISMATCH);
    return;
  }
  const long long t = s_pos;
  const long long j0 = (t - K + 1 > 0) ? t - K + 1 : 0;
  const int nwin = static_cast<int>(t - j0 + 1);
  const int eslot = static_cast<int>(t % K);   // slot of t (and of the evicted t-k)
  const int slot0 = static_cast<int>(j0 % K);  // slot of the first window position
  const bool evict = t >= K;
  const int rslot = static_cast<int>(t % kRing);

  // The ring slot being replaced depends on t: one round trip later,
  // overlapped with the near field.
  const int c4 = tid;  // float4 index within the slice
  const bool ep = c4 < HS / 4;
  const int gi = rank * HS + c4 * 4;
  float4 ring_old = make_float4(0.f, 0.f, 0.f, 0.f);
  if (ep) ring_old = *reinterpret_cast<const float4*>(ring + static_cast<size_t>(rslot) * p.H + gi);

  bool ok = mbar_wait_bounded(bar_in, 0, kMbarPollLimit, p.err);
  for (int i = tid * 4; i < HS; i += kDecodeThreads * 4) {
    float v[4];
    VecLoad<Tin, 4>::run(qraw + i, v);
    *reinterpret_cast<float4*>(qf + i) = make_float4(v[0], v[1], v[2], v[3]);
  }
  __syncthreads();

  // Row of the a-th window position (a = 0 .. nwin-1, position j0+a) for
  // local KV head gg: K_t/V_t from the input copy, older positions from the
  // window (shared or global memory); a == -1 names the evicted key t-k.
  auto wslot = [&](int a) -> int {
    if (a < 0) return eslot;
    const int s2 = slot0 + a;
    return s2 >= K ? s2 - K : s2;
  };
  auto krow = [&](int a, int gg) -> const Tin* {
    if (a == nwin - 1) return kc + gg * D;
    const int sl2 = wslot(a);
    return pl.stage_win ? reinterpret_cast<const Tin*>(wk + sl2 * pl.rec) + gg * D
                        : win_k + (static_cast<size_t>(sl2) * nkv + g_lo + gg) * D;
  };
  auto vrow = [&](int a, int gg) -> const Tin* {
    if (a == nwin - 1) return vc + gg * D;
    const int sl2 = wslot(a);
    return pl.stage_win ? reinterpret_cast<const Tin*>(wv + sl2 * pl.rec) + gg * D
                        : win_v + (static_cast<size_t>(sl2) * nkv + g_lo + gg) * D;
  };

  // (1)-(4) near field per query head [P1 §2.1 eq. O_near]: lane a scores
  // window position j0+a in full (chunks of 32 keys), online softmax across
  // chunks, P·V with lanes over head dims; far field with the evicted key
  // [P1 §2.1 eq. S_t]; x = O_near + alpha_far * S [P1 §2.1 eq. O].
  for (int hh = warp; hh < HPC; hh += NW) {
    const int gg = (h0 + hh) / G - g_lo;
    const float* qh = qf + hh * D;
    float m = -INFINITY, den = 0.f, o[EPL];
#pragma unroll
    for (int e = 0; e < EPL; ++e) o[e] = 0.f;
    for (int base = 0; base < nwin; base += 32) {
      const int cnt = min(32, nwin - base);
      float s = -INFINITY;
      if (lane < cnt) {
        const Tin* kp = krow(base + lane, gg);
        constexpr int VE = Load16<Tin>::N;
        float acc[4] = {0.f, 0.f, 0.f, 0.f};  // independent chains
#pragma unroll
        for (int i = 0; i < D; i += VE) {
          float kv[VE];
          Load16<Tin>::run(kp + i, kv);
#pragma unroll
          for (int e = 0; e < VE; ++e) acc[e & 3] = fmaf(qh[i + e], kv[e], acc[e & 3]);
        }
        s = ((acc[0] + acc[1]) + (acc[2] + acc[3])) * p.score_scale;
      }
      const float mn = fmaxf(m, warp_max(s));
      const float corr = expf(m - mn);
      const float pj = (lane < cnt) ? expf(s - mn) : 0.f;
      den = fmaf(den, corr, warp_sum(pj));
#pragma unroll
      for (int e = 0; e < EPL; ++e) o[e] *= corr;
      for (int c0 = 0; c0 < cnt; c0 += 8) {
        float vv[8][EPL];
#pragma unroll
        for (int u = 0; u < 8; ++u)
          if (c0 + u < cnt) VecLoad<Tin, EPL>::run(vrow(base + c0 + u, gg) + lane * EPL, vv[u]);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const float pc = __shfl_sync(0xffffffffu, pj, (c0 + u) & 31);
          if (c0 + u < cnt) {
#pragma unroll
            for (int e = 0; e < EPL; ++e) o[e] = fmaf(pc, vv[u][e], o[e]);
          }
        }
      }
      m = mn;
    }
    const float inv = 1.f / den;
    float ev[EPL];
    if (evict) VecLoad<Tin, EPL>::run(krow(-1, gg) + lane * EPL, ev);
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      const float s_old = sg[gg * D + lane * EPL + e];
      const float s_new = evict ? ewma(p.gamma_far, s_old, ev[e]) : s_old;
      xs[hh * D + lane * EPL + e] = fmaf(p.alpha_far, s_new, o[e] * inv);
    }
  }
  __syncthreads();

  // (7a) pool partial sums over this slice [P3 §2.1 channel 3]: warp w takes a
  // quarter of the slice, lane j slots j and j+32.
  ok = mbar_wait_bounded(bar_sl, 0, kMbarPollLimit, p.err) && ok;
  {
    const int q4 = HS / NW;  // elements per warp
    const float* x0 = xs + warp * q4;
    const float* r0 = sl + lane * (HS + 4) + warp * q4;
    const float* r1 = sl + (lane + 32) * (HS + 4) + warp * q4;
    float4 a0 = make_float4(0.f, 0.f, 0.f, 0.f), a1 = a0;  // one chain per component
    float ss = 0.f;
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
    if (lane == 0) red[warp * kRedStride + kSlots] = ss;
  }
  __syncthreads();
  if (tid <= kSlots) {
    float acc = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) acc += red[w * kRedStride + tid];
    part[tid] = acc;
  }
  // Partials visible to the cluster; every CTA has finished reading the
  // window slot, S and pos of this stream (its copies have landed).
  cluster.sync();

  // (7b) add the partials of all ranks in rank order (identical in every
  // CTA), softmax(cos/T), weights to shared memory.  Thread i < 65 fetches
  // entry i from every rank (all remote loads in flight), warp 0 finishes.
  if (tid <= kSlots) {
    float v[kMaxCluster];
#pragma unroll
    for (int r = 0; r < kMaxCluster; ++r)
      v[r] = (r < p.CS) ? cluster.map_shared_rank(part, r)[tid] : 0.f;
    float acc = 0.f;
#pragma unroll
    for (int r = 0; r < kMaxCluster; ++r) acc += v[r];
    red[tid] = acc;  // per-warp partials are no longer needed
  }
  cluster_arrive();  // done with the peers' shared memory
  __syncthreads();
  if (warp == 0) {
    const float d0 = red[lane], d1 = red[lane + 32], ss = red[kSlots];
    const float nx = fmaxf(sqrtf(ss), kNormFloor);
    const float c0 = d0 / (nx * nrm0) * p.inv_temp;
    const float c1 = d1 / (nx * nrm1) * p.inv_temp;
    const float mx = warp_max(fmaxf(c0, c1));
    const float e0 = expf(c0 - mx), e1 = expf(c1 - mx);
    const float inv = 1.f / warp_sum(e0 + e1);
    wts[lane] = e0 * inv;
    wts[lane + 32] = e1 * inv;
  }
  __syncthreads();

  // (5)(6)(7c)(8): ring, field, semantic mix, fusion, clip, scale, output.
  if (ep && ok) {
    const int i = c4 * 4;
    float4 se = make_float4(0.f, 0.f, 0.f, 0.f), so = se;  // even / odd slots
#pragma unroll 16
    for (int j = 0; j < kSlots; j += 2) {
      const float4 s4 = *reinterpret_cast<const float4*>(sl + j * (HS + 4) + i);
      const float4 t4 = *reinterpret_cast<const float4*>(sl + (j + 1) * (HS + 4) + i);
      const float w0 = wts[j], w1 = wts[j + 1];
      se.x = fmaf(w0, s4.x, se.x); se.y = fmaf(w0, s4.y, se.y);
      se.z = fmaf(w0, s4.z, se.z); se.w = fmaf(w0, s4.w, se.w);
      so.x = fmaf(w1, t4.x, so.x); so.y = fmaf(w1, t4.y, so.y);
      so.z = fmaf(w1, t4.z, so.z); so.w = fmaf(w1, t4.w, so.w);
    }
    const float4 sem = make_float4(se.x + so.x, se.y + so.y, se.z + so.z, se.w + so.w);
    const float4 x4 = *reinterpret_cast<const float4*>(xs + i);
    const float4 rs4 = *reinterpret_cast<const float4*>(rsm + i);
    const float4 f4 = *reinterpret_cast<const float4*>(fld + i);
    const float xv[4] = {x4.x, x4.y, x4.z, x4.w};
    const float ov[4] = {ring_old.x, ring_old.y, ring_old.z, ring_old.w};
    float rv[4] = {rs4.x, rs4.y, rs4.z, rs4.w};
    float fv[4] = {f4.x, f4.y, f4.z, f4.w};
    const float sv[4] = {sem.x, sem.y, sem.z, sem.w};
    float outv[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      rv[e] = (rv[e] - ov[e]) + xv[e];          // ring sum after storing x_t
      fv[e] = ewma(p.ema_gamma, fv[e], xv[e]);  // EMA field
      float u = rv[e] * (1.0f / kRing) + 0.5f * fv[e] + 0.5f * sv[e];
      u = fminf(fmaxf(u, -p.clip_eps), p.clip_eps);
      outv[e] = fmaf(a_l, u, xv[e]);
    }
    *reinterpret_cast<float4*>(ring + static_cast<size_t>(rslot) * p.H + gi) = x4;
    *reinterpret_cast<float4*>(ring_sum + gi) = make_float4(rv[0], rv[1], rv[2], rv[3]);
    *reinterpret_cast<float4*>(field + gi) = make_float4(fv[0], fv[1], fv[2], fv[3]);
    *reinterpret_cast<float4*>(p.out + stream * p.H + gi) = make_float4(outv[0], outv[1], outv[2], outv[3]);
  }

  // (1)(2) write-back of the KV heads this CTA owns, from the staged copies:
  // S with the evicted key, then K_t, V_t into slot t mod k.  Every CTA of
  // the cluster has read the old values (first cluster barrier above).
  if (ok) {
    const int n_own = g_hi - own_lo + 1;
    for (int idx = tid; idx < n_own * D; idx += kDecodeThreads) {
      const int gg = own_lo - g_lo + idx / D;
      const int i = idx % D;
      float s = sg[gg * D + i];
      if (evict) s = ewma(p.gamma_far, s, to_f32<Tin>(krow(-1, gg)[i]));
      const size_t wo = (static_cast<size_t>(eslot) * nkv + g_lo + gg) * D + i;
      far[(g_lo + gg) * D + i] = s;
      win_k[wo] = kc[gg * D + i];
      win_v[wo] = vc[gg * D + i];
    }
    if (rank == 0 && tid == 0) *reinterpret_cast<long long*>(blk + p.so.pos) = t + 1;
  }

  // No CTA may leave while a peer can still read its `part` array.
  cluster_wait();
}

template <typename Tin, int D>
cudaError_t launch_t(const DecodeParams& p, cudaStream_t s) {
  const DecodePlan pl = decode_plan(p.HPC, D, static_cast<int>(sizeof(Tin)), p.NGm, p.K, p.smem_budget);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.CS, p.B, p.L);
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
  return cudaLaunchKernelEx(&cfg, decode_kernel<Tin, D>, p);
}

template <typename Tin, int D>
cudaError_t prepare_t(int optin) {
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, decode_kernel<Tin, D>);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(decode_kernel<Tin, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             optin - static_cast<int>(fa.sharedSizeBytes));
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(decode_kernel<Tin, D>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  return e;
}

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
  if (cudaOccupancyMaxActiveClusters(&n, decode_kernel<Tin, D>, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}

}  // namespace

// Shared memory of one decode CTA; the window is staged when it fits in
// `budget` bytes together with everything else.
size_t decode_smem_bytes(int HPC, int head_dim, int esz, int NGm, int K, int budget) {
  return static_cast<size_t>(decode_plan(HPC, head_dim, esz, NGm, K, budget).total);
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
