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
// bandwidth.  The slot slice (the largest read) is staged into shared memory
// by the bulk-copy engine before the kernel waits on its predecessor
// (programmatic dependent launch: slots are constant), and every other load
// is issued before its first use, so a step costs about two memory round
// trips plus one cluster exchange.
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

constexpr int NW = kDecodeThreads / 32;
constexpr int kRedStride = kSlots + 4;  // per-warp partials: 64 dots + |x|^2

struct DecodeSmem {
  int sl, qs, xs, red, part, wts, total;
};

// Shared-memory plan in floats; slot rows are padded by 4 floats so that
// lanes reading different rows at the same column hit distinct banks.
__host__ __device__ inline DecodeSmem decode_smem(int HS, int HPC, int D) {
  DecodeSmem s;
  s.sl = 4;  // the mbarrier lives in the first 16 bytes
  s.qs = s.sl + kSlots * (HS + 4);
  s.xs = s.qs + HPC * D;
  s.red = s.xs + HS;
  s.part = s.red + NW * kRedStride;
  s.wts = s.part + kRedStride;
  s.total = s.wts + kSlots;
  return s;
}

template <typename Tin, int D>
__global__ void __launch_bounds__(kDecodeThreads)
decode_kernel(const DecodeParams p) {
  constexpr int EPL = D / 32;  // elements of a head row per lane
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = static_cast<int>(cluster.block_rank());
  const int b = blockIdx.y, l = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int HS = p.HPC * D;

  extern __shared__ __align__(16) float smem[];
  const DecodeSmem sp = decode_smem(HS, p.HPC, D);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem);
  float* sl = smem + sp.sl;      // [64][HS+4] slot slice
  float* qs = smem + sp.qs;      // [HPC][D]   queries of this CTA's heads
  float* xs = smem + sp.xs;      // [HS]       x_t, this CTA's slice
  float* red = smem + sp.red;    // [NW][68]   per-warp pool partials
  float* part = smem + sp.part;  // [68]       CTA pool partials
  float* wts = smem + sp.wts;    // [64]       pool softmax weights
  __shared__ long long s_pos;
  __shared__ int s_ok;

  if (tid == 0) {
    mbar_init(bar, 1);
    mbar_fence_init();
  }
  __syncthreads();
  pdl_trigger();

  // Slot slice: constant since sfa_init, so it may be fetched before the
  // previous kernel of the stream has finished.
  const float* slot_base = p.slots + static_cast<size_t>(l) * kSlots * p.H + static_cast<size_t>(rank) * HS;
  if (warp == 0) {
    if (lane == 0) mbar_arrive_expect_tx(bar, kSlots * HS * 4u);
    __syncwarp();
    for (int j = lane; j < kSlots; j += 32)
      bulk_g2s(sl + j * (HS + 4), slot_base + static_cast<size_t>(j) * p.H, HS * 4u, bar);
  }

  pdl_wait();  // state and inputs may be written by the previous kernel

  const long long stream = static_cast<long long>(l) * p.B + b;
  unsigned char* blk = p.state + kHeaderBytes + stream * p.so.stride;
  if (tid == 0) {
    const StateHeader* hdr = reinterpret_cast<const StateHeader*>(p.state);
    s_ok = (hdr->magic == kMagic && hdr->cfg_hash == p.cfg_hash && hdr->batch == p.B &&
            hdr->n_layers == p.L);
    s_pos = *reinterpret_cast<const long long*>(blk + p.so.pos);
  }
  // queries of this CTA's heads -> shared memory (fp32)
  const Tin* qin = static_cast<const Tin*>(p.q) + (stream * p.nq + static_cast<long long>(rank) * p.HPC) * D;
  for (int i = tid * EPL; i < HS; i += kDecodeThreads * EPL) {
    float v[EPL];
    VecLoad<Tin, EPL>::run(qin + i, v);
#pragma unroll
    for (int e = 0; e < EPL; ++e) qs[i + e] = v[e];
  }
  __syncthreads();
  if (!s_ok) {  // the same header for every CTA: the whole grid leaves here
    mbar_wait_bounded(bar, 0, kMbarPollLimit, p.err);  // no copy may land after exit
    if (tid == 0 && rank == 0 && b == 0 && l == 0) latch_error(p.err, SFA_ERR_STATE_MISMATCH);
    return;
  }
  const long long t = s_pos;

  Tin* win_k = reinterpret_cast<Tin*>(blk + p.so.win_k);
  Tin* win_v = reinterpret_cast<Tin*>(blk + p.so.win_v);
  float* far = reinterpret_cast<float*>(blk + p.so.far);
  float* field = reinterpret_cast<float*>(blk + p.so.field);
  float* ring_sum = reinterpret_cast<float*>(blk + p.so.ring_sum);
  float* ring = reinterpret_cast<float*>(blk + p.so.ring);
  const Tin* kin = static_cast<const Tin*>(p.k) + stream * p.nkv * D;
  const Tin* vin = static_cast<const Tin*>(p.v) + stream * p.nkv * D;
  const int K = p.K;
  const long long j0 = (t - K + 1 > 0) ? t - K + 1 : 0;
  const int nwin = static_cast<int>(t - j0 + 1);
  const int eslot = static_cast<int>(t % K);
  const bool evict = t >= K;
  const int rslot = static_cast<int>(t % kRing);
  const int h0 = rank * p.HPC;

  // Epilogue operands of this thread's float4 of the slice, in flight
  // during the near field.
  const int c4 = tid;  // float4 index within the slice
  const bool ep = c4 < HS / 4;
  const int gi = rank * HS + c4 * 4;
  float4 ring_old = make_float4(0.f, 0.f, 0.f, 0.f), rs4 = ring_old, f4 = ring_old;
  if (ep) {
    ring_old = *reinterpret_cast<const float4*>(ring + static_cast<size_t>(rslot) * p.H + gi);
    rs4 = *reinterpret_cast<const float4*>(ring_sum + gi);
    f4 = *reinterpret_cast<const float4*>(field + gi);
  }

  // (1)-(4) near field per query head [P1 §2.1 eq. O_near]: lane a scores
  // window position j0+a in full (keys in chunks of 32), online softmax across
  // chunks, then P·V with lanes over head dims; far field S with the evicted
  // key [P1 §2.1 eq. S_t]; x = O_near + alpha_far * S [P1 §2.1 eq. O].
  for (int hh = warp; hh < p.HPC; hh += NW) {
    const int h = h0 + hh;
    const int g = h / p.G;
    const float* qh = qs + hh * D;
    float sv[EPL], evv[EPL];
    VecLoad<float, EPL>::run(far + g * D + lane * EPL, sv);
    if (evict) VecLoad<Tin, EPL>::run(win_k + (static_cast<size_t>(eslot) * p.nkv + g) * D + lane * EPL, evv);
    float m = -INFINITY, den = 0.f, o[EPL];
#pragma unroll
    for (int e = 0; e < EPL; ++e) o[e] = 0.f;
    for (int base = 0; base < nwin; base += 32) {
      const int cnt = min(32, nwin - base);
      const long long j = j0 + base + lane;
      float s = -INFINITY;
      if (lane < cnt) {
        const Tin* kp = (j == t) ? kin + g * D
                                 : win_k + (static_cast<size_t>(j % K) * p.nkv + g) * D;
        constexpr int VE = Load16<Tin>::N;
        float acc = 0.f;
#pragma unroll
        for (int i = 0; i < D; i += VE) {
          float kv[VE];
          Load16<Tin>::run(kp + i, kv);
#pragma unroll
          for (int e = 0; e < VE; ++e) acc = fmaf(qh[i + e], kv[e], acc);
        }
        s = acc * p.score_scale;
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
        for (int u = 0; u < 8; ++u) {
          const int c = c0 + u;
          if (c < cnt) {
            const long long jc = j0 + base + c;
            const Tin* vp = (jc == t) ? vin + g * D
                                      : win_v + (static_cast<size_t>(jc % K) * p.nkv + g) * D;
            VecLoad<Tin, EPL>::run(vp + lane * EPL, vv[u]);
          }
        }
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
#pragma unroll
    for (int e = 0; e < EPL; ++e) {
      const float s_new = evict ? ewma(p.gamma_far, sv[e], evv[e]) : sv[e];
      xs[hh * D + lane * EPL + e] = fmaf(p.alpha_far, s_new, o[e] * inv);
    }
  }
  __syncthreads();

  // (7a) pool partial sums over this slice [P3 §2.1 channel 3]: warp w takes a
  // quarter of the slice, lane j slots j and j+32.
  const bool slots_ok = mbar_wait_bounded(bar, 0, kMbarPollLimit, p.err);
  {
    const int q4 = HS / NW;  // elements per warp
    const float* x0 = xs + warp * q4;
    const float* r0 = sl + lane * (HS + 4) + warp * q4;
    const float* r1 = sl + (lane + 32) * (HS + 4) + warp * q4;
    float d0 = 0.f, d1 = 0.f, ss = 0.f;
    for (int e = 0; e < q4; e += 4) {
      const float4 xv = *reinterpret_cast<const float4*>(x0 + e);
      const float4 a = *reinterpret_cast<const float4*>(r0 + e);
      const float4 c = *reinterpret_cast<const float4*>(r1 + e);
      d0 = fmaf(xv.x, a.x, fmaf(xv.y, a.y, fmaf(xv.z, a.z, fmaf(xv.w, a.w, d0))));
      d1 = fmaf(xv.x, c.x, fmaf(xv.y, c.y, fmaf(xv.z, c.z, fmaf(xv.w, c.w, d1))));
    }
    for (int e = lane; e < q4; e += 32) ss = fmaf(x0[e], x0[e], ss);
    ss = warp_sum(ss);
    red[warp * kRedStride + lane] = d0;
    red[warp * kRedStride + lane + 32] = d1;
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
  if (ep && slots_ok) {
    const float a_l = p.alpha_layer[l];
    const int i = c4 * 4;
    float4 sem = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 16
    for (int j = 0; j < kSlots; ++j) {
      const float4 s4 = *reinterpret_cast<const float4*>(sl + j * (HS + 4) + i);
      const float w = wts[j];
      sem.x = fmaf(w, s4.x, sem.x);
      sem.y = fmaf(w, s4.y, sem.y);
      sem.z = fmaf(w, s4.z, sem.z);
      sem.w = fmaf(w, s4.w, sem.w);
    }
    const float4 x4 = *reinterpret_cast<const float4*>(xs + i);
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

  // (1)(2) write-back of the KV heads this CTA owns: S with the evicted key,
  // then K_t, V_t into slot t mod k.  Safe after the barrier above.
  if (slots_ok) {
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
    if (rank == 0 && tid == 0) *reinterpret_cast<long long*>(blk + p.so.pos) = t + 1;
  }

  // No CTA may leave while a peer can still read its `part` array.
  cluster.sync();
}

template <typename Tin, int D>
cudaError_t launch_t(const DecodeParams& p, cudaStream_t s) {
  const size_t smem = static_cast<size_t>(decode_smem(p.HPC * D, p.HPC, D).total) * sizeof(float);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.CS, p.B, p.L);
  cfg.blockDim = dim3(kDecodeThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
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

}  // namespace

size_t decode_smem_bytes(int HPC, int head_dim) {
  return static_cast<size_t>(decode_smem(HPC * head_dim, HPC, head_dim).total) * sizeof(float);
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
