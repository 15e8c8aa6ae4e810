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
// Ordering.  The window slot t mod k and the far state S are read by every
// CTA that needs that KV head, and written by one owner CTA (the one holding
// the group's first query head) only after the first cluster barrier, when
// all reads are done.  Ring, ring-sum and field elements belong to exactly
// one CTA.  The stream position is read at entry and advanced by rank 0
// after the first barrier.
#include <cooperative_groups.h>
#include <cuda_bf16.h>

#include "sfa_common.cuh"

namespace cg = cooperative_groups;

namespace sfa {
namespace {

template <typename Tin, int D>
__global__ void __launch_bounds__(kDecodeThreads)
decode_kernel(const DecodeParams p) {
  constexpr int EPL = D / 32;  // elements of a head row per lane
  constexpr int NW = kDecodeThreads / 32;
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = static_cast<int>(cluster.block_rank());
  const int b = blockIdx.y, l = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  __shared__ __align__(16) float xs[kMaxSlice];  // x_t, this CTA's slice
  __shared__ float part[kSlots + 1];              // partial x·slot_j and |x|^2
  __shared__ float wts[kSlots];                   // pool softmax weights
  __shared__ float red[NW];
  __shared__ int s_ok;

  // The header is read by every CTA, so a mismatch is seen uniformly and
  // all CTAs of every cluster leave before any cluster barrier.
  if (tid == 0) {
    const StateHeader* hdr = reinterpret_cast<const StateHeader*>(p.state);
    s_ok = (hdr->magic == kMagic && hdr->cfg_hash == p.cfg_hash && hdr->batch == p.B &&
            hdr->n_layers == p.L);
  }
  __syncthreads();
  if (!s_ok) {
    if (tid == 0 && rank == 0 && b == 0 && l == 0) latch_error(p.err, SFA_ERR_STATE_MISMATCH);
    return;
  }

  const long long stream = static_cast<long long>(l) * p.B + b;
  unsigned char* blk = p.state + kHeaderBytes + stream * p.so.stride;
  const long long t = *reinterpret_cast<const long long*>(blk + p.so.pos);
  Tin* win_k = reinterpret_cast<Tin*>(blk + p.so.win_k);
  Tin* win_v = reinterpret_cast<Tin*>(blk + p.so.win_v);
  float* far = reinterpret_cast<float*>(blk + p.so.far);
  float* field = reinterpret_cast<float*>(blk + p.so.field);
  float* ring_sum = reinterpret_cast<float*>(blk + p.so.ring_sum);
  float* ring = reinterpret_cast<float*>(blk + p.so.ring);

  const int HS = p.HPC * D;
  const int h0 = rank * p.HPC;
  const Tin* qin = static_cast<const Tin*>(p.q) + stream * p.nq * D;
  const Tin* kin = static_cast<const Tin*>(p.k) + stream * p.nkv * D;
  const Tin* vin = static_cast<const Tin*>(p.v) + stream * p.nkv * D;
  const int K = p.K;
  const long long j0 = (t - K + 1 > 0) ? t - K + 1 : 0;
  const int nwin = static_cast<int>(t - j0 + 1);
  const int eslot = static_cast<int>(t % K);
  const bool evict = t >= K;

  // (1)-(4): near field per query head (one warp per head, online softmax
  // with warp-shuffle reductions), far-field EWMA with the evicted key, and
  // the dual-channel sum x = O_near + alpha_far * S  [P1 §2.1].
  for (int hh = warp; hh < p.HPC; hh += NW) {
    const int h = h0 + hh;
    const int g = h / p.G;
    float qv[EPL];
    VecLoad<Tin, EPL>::run(qin + h * D + lane * EPL, qv);
    float m = -INFINITY, den = 0.f, o[EPL];
#pragma unroll
    for (int e = 0; e < EPL; ++e) o[e] = 0.f;
    for (int a = 0; a < nwin; ++a) {
      const long long j = j0 + a;
      const Tin* kp;
      const Tin* vp;
      if (j == t) {  // the current token comes from the input, not the state
        kp = kin + g * D;
        vp = vin + g * D;
      } else {
        const size_t off = (static_cast<size_t>(j % K) * p.nkv + g) * D;
        kp = win_k + off;
        vp = win_v + off;
      }
      float kv[EPL], vv[EPL];
      VecLoad<Tin, EPL>::run(kp + lane * EPL, kv);
      VecLoad<Tin, EPL>::run(vp + lane * EPL, vv);
      float s = 0.f;
#pragma unroll
      for (int e = 0; e < EPL; ++e) s = fmaf(qv[e], kv[e], s);
      s = warp_sum(s) * p.score_scale;
      const float mn = fmaxf(m, s);
      const float corr = expf(m - mn);
      const float pj = expf(s - mn);
      den = fmaf(den, corr, pj);
#pragma unroll
      for (int e = 0; e < EPL; ++e) o[e] = fmaf(o[e], corr, pj * vv[e]);
      m = mn;
    }
    const float inv = 1.f / den;
    float sv[EPL];
    VecLoad<float, EPL>::run(far + g * D + lane * EPL, sv);
    if (evict) {
      float ev[EPL];
      VecLoad<Tin, EPL>::run(win_k + (static_cast<size_t>(eslot) * p.nkv + g) * D + lane * EPL, ev);
#pragma unroll
      for (int e = 0; e < EPL; ++e) sv[e] = ewma(p.gamma_far, sv[e], ev[e]);
    }
#pragma unroll
    for (int e = 0; e < EPL; ++e) xs[hh * D + lane * EPL + e] = fmaf(p.alpha_far, sv[e], o[e] * inv);
  }
  __syncthreads();

  // (7a) pool partial sums over this slice [P3 §2.1 channel 3].
  const float* slot_base = p.slots + static_cast<size_t>(l) * kSlots * p.H + static_cast<size_t>(rank) * HS;
  for (int j = warp; j < kSlots; j += NW) {
    const float* sr = slot_base + static_cast<size_t>(j) * p.H;
    float acc = 0.f;
    for (int i = lane * 4; i < HS; i += 128) {
      const float4 s4 = __ldg(reinterpret_cast<const float4*>(sr + i));
      const float4 x4 = *reinterpret_cast<const float4*>(xs + i);
      acc = fmaf(s4.x, x4.x, acc);
      acc = fmaf(s4.y, x4.y, acc);
      acc = fmaf(s4.z, x4.z, acc);
      acc = fmaf(s4.w, x4.w, acc);
    }
    acc = warp_sum(acc);
    if (lane == 0) part[j] = acc;
  }
  {
    float ss = 0.f;
    for (int i = tid; i < HS; i += kDecodeThreads) ss = fmaf(xs[i], xs[i], ss);
    ss = warp_sum(ss);
    if (lane == 0) red[warp] = ss;
    __syncthreads();
    if (tid == 0) {
      float tot = 0.f;
      for (int w = 0; w < NW; ++w) tot += red[w];
      part[kSlots] = tot;
    }
  }
  // Partials visible to the cluster; every CTA has finished reading the
  // window slot, S and pos of this stream.
  cluster.sync();

  // (7b) add the partials of all ranks in rank order (identical in every
  // CTA), softmax(cos/T), weights to shared memory.
  if (warp == 0) {
    float d0 = 0.f, d1 = 0.f, ss = 0.f;
    for (int r = 0; r < p.CS; ++r) {
      const float* rp = cluster.map_shared_rank(part, r);
      d0 += rp[lane];
      d1 += rp[lane + 32];
      ss += rp[kSlots];
    }
    const float nx = fmaxf(sqrtf(ss), kNormFloor);
    const float* nrm = p.slot_norm + static_cast<size_t>(l) * kSlots;
    const float c0 = d0 / (nx * nrm[lane]) * p.inv_temp;
    const float c1 = d1 / (nx * nrm[lane + 32]) * p.inv_temp;
    const float mx = warp_max(fmaxf(c0, c1));
    const float e0 = expf(c0 - mx), e1 = expf(c1 - mx);
    const float inv = 1.f / warp_sum(e0 + e1);
    wts[lane] = e0 * inv;
    wts[lane + 32] = e1 * inv;
  }
  __syncthreads();

  // (5)(6)(7c)(8): ring, field, semantic mix, fusion, clip, scale, output.
  const float a_l = p.alpha_layer[l];
  const int rslot = static_cast<int>(t % kRing);
  float* out = p.out + stream * p.H;
  for (int c4 = tid; c4 < HS / 4; c4 += kDecodeThreads) {
    const int i = c4 * 4;
    const int gi = rank * HS + i;
    float4 sem = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
    for (int j = 0; j < kSlots; ++j) {
      const float4 s4 = __ldg(reinterpret_cast<const float4*>(slot_base + static_cast<size_t>(j) * p.H + i));
      const float w = wts[j];
      sem.x = fmaf(w, s4.x, sem.x);
      sem.y = fmaf(w, s4.y, sem.y);
      sem.z = fmaf(w, s4.z, sem.z);
      sem.w = fmaf(w, s4.w, sem.w);
    }
    const float4 x4 = *reinterpret_cast<const float4*>(xs + i);
    float4* rp = reinterpret_cast<float4*>(ring + static_cast<size_t>(rslot) * p.H + gi);
    float4* rsp = reinterpret_cast<float4*>(ring_sum + gi);
    float4* fp = reinterpret_cast<float4*>(field + gi);
    const float4 old = *rp;
    float4 rs = *rsp;
    float4 f = *fp;
    const float xv[4] = {x4.x, x4.y, x4.z, x4.w};
    const float ov[4] = {old.x, old.y, old.z, old.w};
    float rv[4] = {rs.x, rs.y, rs.z, rs.w};
    float fv[4] = {f.x, f.y, f.z, f.w};
    const float sv[4] = {sem.x, sem.y, sem.z, sem.w};
    float outv[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      rv[e] = (rv[e] - ov[e]) + xv[e];               // ring sum after storing x_t
      fv[e] = ewma(p.ema_gamma, fv[e], xv[e]);       // EMA field
      float u = rv[e] * (1.0f / kRing) + 0.5f * fv[e] + 0.5f * sv[e];
      u = fminf(fmaxf(u, -p.clip_eps), p.clip_eps);
      outv[e] = fmaf(a_l, u, xv[e]);
    }
    *rp = x4;
    *rsp = make_float4(rv[0], rv[1], rv[2], rv[3]);
    *fp = make_float4(fv[0], fv[1], fv[2], fv[3]);
    *reinterpret_cast<float4*>(out + gi) = make_float4(outv[0], outv[1], outv[2], outv[3]);
  }

  // (1)(2) write-back of the KV heads this CTA owns: S with the evicted key,
  // then K_t, V_t into slot t mod k.  Safe after the barrier above.
  {
    const int own_lo = (h0 + p.G - 1) / p.G;
    const int own_hi = (h0 + p.HPC - 1) / p.G;
    const int n_own = own_hi - own_lo + 1;
    for (int idx = tid; idx < n_own * D; idx += kDecodeThreads) {
      const int g = own_lo + idx / D;
      const int i = idx % D;
      const size_t wo = (static_cast<size_t>(eslot) * p.nkv + g) * D + i;
      float s = far[g * D + i];
      if (evict) s = ewma(p.gamma_far, s, to_f32<Tin>(win_k[wo]));
      far[g * D + i] = s;
      win_k[wo] = kin[g * D + i];
      win_v[wo] = vin[g * D + i];
    }
  }
  if (rank == 0 && tid == 0) *reinterpret_cast<long long*>(blk + p.so.pos) = t + 1;

  // No CTA may leave while a peer can still read its `part` array.
  cluster.sync();
}

template <typename Tin, int D>
cudaError_t launch_t(const DecodeParams& p, cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.CS, p.B, p.L);
  cfg.blockDim = dim3(kDecodeThreads, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = p.CS;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode_kernel<Tin, D>, p);
}

}  // namespace

cudaError_t launch_decode(const DecodeParams& p, int in_dtype, int head_dim, cudaStream_t s) {
  if (in_dtype == SFA_F32) {
    return head_dim == 64 ? launch_t<float, 64>(p, s) : launch_t<float, 128>(p, s);
  }
  return head_dim == 64 ? launch_t<__nv_bfloat16, 64>(p, s) : launch_t<__nv_bfloat16, 128>(p, s);
}

}  // namespace sfa
