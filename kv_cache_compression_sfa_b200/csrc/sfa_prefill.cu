// sfa_prefill.cu — SFA prefill: n tokens per (layer, sequence) stream, in
// parallel over token tiles.
//
// Sources (web pages):
//   [P1] "Signal Field Attention (SFA)：8KB代码实现4.16倍推理加速与248倍内存压缩"
//        §2.1 eqs. O_near, S_t, O; §2.2 O(k·d) window state.
//   [P3] "Dalin Soma SFA基于信号场注意力机制的神经网络推理加速框架"
//        §2.1 channels 1–3, §2.2 fusion, clip and alpha_layer, §2.4 ring mean.
//
// Work unit: one tile of kTile consecutive tokens of one stream, served by a
// cluster of CS CTAs; CTA `rank` owns query heads [rank*HPC, (rank+1)*HPC)
// and hence hidden slice [rank*HS, (rank+1)*HS).  Tiles get an ordered ticket
// from a global counter (tile-major over streams), so a tile only ever waits
// on tiles with smaller tickets, which are already running or done.
//
// The method's three recurrences become parallel scans across tiles:
//   * far-field EWMA S (per KV head, depends on keys only): each tile
//     publishes its local aggregate A and the carried-in value is found by a
//     decoupled look-back over predecessors (S_end = gamma^m * S_start + A);
//   * EMA field (per hidden element, depends on x): same scheme;
//   * ring mean: a sliding 16-token sum; the 15 rows of x before a tile come
//     from its predecessor's published tail rows (or from the state ring).
// Every wait is bounded; a wait that runs out latches
// SFA_ERR_DEVICE_TIMEOUT and the kernel still finishes.
//
// The semantic pool needs |x| and x·slot_j over all of hidden: partial sums
// of the slice are reduce-scattered across the cluster through distributed
// shared memory (rank r finishes tokens r, r+CS, ...) and the softmax
// weights are written back into every CTA's shared memory.
#include <cooperative_groups.h>
#include <cuda_bf16.h>

#include "sfa_common.cuh"

namespace cg = cooperative_groups;

namespace sfa {
namespace {

constexpr int kPartStride = kSlots + 1;  // 64 partial dots + |x|^2 per token
constexpr int kChunk = 32;               // hidden elements per staged slot chunk

struct SmemPlan {
  int xs, halo, part, wts, sst, sagg, fcar, schunk, total_floats;
};

__host__ __device__ inline SmemPlan plan_smem(int HPC, int D) {
  const int HS = HPC * D;
  SmemPlan s;
  s.xs = 0;
  s.halo = s.xs + kTile * HS;
  s.part = s.halo + kHalo * HS;
  s.wts = s.part + kTile * kPartStride;
  s.sst = s.wts + kTile * kSlots;
  s.sagg = s.sst + (HPC + 1) * D;
  s.fcar = s.sagg + (HPC + 1) * D;
  s.schunk = s.fcar + HS;
  s.total_floats = s.schunk + kSlots * (kChunk + 1);
  s.total_floats = (s.total_floats + 3) & ~3;
  return s;
}

template <typename Tin>
struct StreamIO {
  const Tin* kin;   // this stream's input keys   [n][nkv][D]
  const Tin* vin;
  const Tin* win_k; // this stream's window slots [K][nkv][D]
  long long pos0;
  int nkv, K, D;
  // Key row of absolute position j (j >= 0): from the input if it belongs to
  // this call, else from the window slot j mod k (the state holds positions
  // pos0-k .. pos0-1).
  __device__ __forceinline__ const Tin* key(long long j, int g) const {
    return (j >= pos0) ? kin + ((j - pos0) * nkv + g) * D
                       : win_k + ((j % K) * nkv + g) * D;
  }
};

template <typename Tin, int D>
__global__ void __launch_bounds__(kPrefillThreads, 1)
prefill_kernel(const PrefillParams p) {
  constexpr int EPL = D / 32;
  constexpr int NT = kPrefillThreads;
  constexpr int NW = NT / 32;
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = static_cast<int>(cluster.block_rank());
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  extern __shared__ __align__(16) float smem[];
  const SmemPlan sp = plan_smem(p.HPC, D);
  const int HS = p.HPC * D;
  float* xs = smem + sp.xs;        // [kTile][HS]  x of this tile's tokens
  float* halo = smem + sp.halo;    // [15][HS]     x of the 15 tokens before
  float* part = smem + sp.part;    // [kTile][65]  partial pool sums
  float* wts = smem + sp.wts;      // [kTile][64]  pool weights
  float* sst = smem + sp.sst;      // [NG][D]      S carried in, then S at tile end
  float* sagg = smem + sp.sagg;    // [NG][D]      this tile's S aggregate
  float* fcar = smem + sp.fcar;    // [HS]         field carried in
  float* schunk = smem + sp.schunk;// [64][33]     staged slot chunk

  __shared__ unsigned long long s_ticket;
  __shared__ unsigned s_flag;
  __shared__ int s_ok;

  // ---- ticket: the tile this cluster serves ----------------------------
  if (rank == 0 && tid == 0) s_ticket = atomicAdd(reinterpret_cast<unsigned long long*>(p.ws), 1ull);
  if (tid == 0) {
    const StateHeader* hdr = reinterpret_cast<const StateHeader*>(p.state);
    s_ok = (hdr->magic == kMagic && hdr->cfg_hash == p.cfg_hash && hdr->batch == p.B &&
            hdr->n_layers == p.L);
  }
  cluster.sync();
  const long long ticket = static_cast<long long>(*cluster.map_shared_rank(&s_ticket, 0));
  if (!s_ok) {  // uniform over the whole grid: every CTA reads the same header
    if (tid == 0 && rank == 0 && ticket == 0) latch_error(p.err, SFA_ERR_STATE_MISMATCH);
    cluster.sync();  // rank 0's s_ticket must outlive the peers' reads
    return;
  }
  const long long tile = ticket / p.n_streams;
  const int stream = static_cast<int>(ticket % p.n_streams);
  const int l = stream / p.B;
  const bool first = (tile == 0);
  const bool last = (tile == p.tiles_per_stream - 1);
  const bool publish = (ticket != p.withhold_tile);

  unsigned char* blk = p.state + kHeaderBytes + static_cast<long long>(stream) * p.so.stride;
  const long long pos0 = *reinterpret_cast<const volatile long long*>(blk + p.so.pos);
  Tin* win_k = reinterpret_cast<Tin*>(blk + p.so.win_k);
  Tin* win_v = reinterpret_cast<Tin*>(blk + p.so.win_v);
  float* far = reinterpret_cast<float*>(blk + p.so.far);
  float* field = reinterpret_cast<float*>(blk + p.so.field);
  float* ring_sum = reinterpret_cast<float*>(blk + p.so.ring_sum);
  float* ring = reinterpret_cast<float*>(blk + p.so.ring);

  const long long t0 = pos0 + tile * kTile;                 // first position of the tile
  const int Tt = static_cast<int>(min(static_cast<long long>(kTile), p.n - tile * kTile));
  const int K = p.K, G = p.G, nkv = p.nkv;
  const int h0 = rank * p.HPC;
  const int g_lo = h0 / G, g_hi = (h0 + p.HPC - 1) / G;
  const int NG = g_hi - g_lo + 1;
  const int own_lo = (h0 + G - 1) / G;                       // KV heads this CTA publishes
  const float gf = p.gamma_far, ge = p.ema_gamma;

  const long long in_row0 = static_cast<long long>(stream) * p.n;  // first input row of the stream
  StreamIO<Tin> io;
  io.kin = static_cast<const Tin*>(p.k) + in_row0 * nkv * D;
  io.vin = static_cast<const Tin*>(p.v) + in_row0 * nkv * D;
  io.win_k = win_k;
  io.pos0 = pos0;
  io.nkv = nkv;
  io.K = K;
  io.D = D;
  const Tin* qin = static_cast<const Tin*>(p.q) + in_row0 * p.nq * D;

  unsigned* flags_s = reinterpret_cast<unsigned*>(p.ws + p.ws_flags_s);
  unsigned* flags_f = reinterpret_cast<unsigned*>(p.ws + p.ws_flags_f);
  float* agg_s = reinterpret_cast<float*>(p.ws + p.ws_agg_s);
  float* incl_s = reinterpret_cast<float*>(p.ws + p.ws_incl_s);
  float* agg_f = reinterpret_cast<float*>(p.ws + p.ws_agg_f);
  float* incl_f = reinterpret_cast<float*>(p.ws + p.ws_incl_f);
  float* halo_ws = reinterpret_cast<float*>(p.ws + p.ws_halo);

  // Evictions inside a full or partial tile starting at absolute position a.
  auto evictions = [&](long long a, int len) -> int {
    const long long lo = a > K ? a : static_cast<long long>(K);
    const long long hi = a + len;
    return hi > lo ? static_cast<int>(hi - lo) : 0;
  };

  // ---- (A) far field: local aggregate of the keys leaving the window ------
  // [P1 §2.1 eq. S_t], key leaving at position t is K_{t-k}.
  for (int idx = tid; idx < NG * D; idx += NT) {
    const int gg = idx / D, i = idx % D, g = g_lo + gg;
    float a = 0.f, mul = 1.f;
    for (int r = 0; r < Tt; ++r) {
      const long long pt = t0 + r;
      if (pt >= K) {
        a = ewma(gf, a, to_f32<Tin>(io.key(pt - K, g)[i]));
        mul *= gf;
      }
    }
    sagg[idx] = a;
    if (first) {  // carry-in is the state's S; the tile's inclusive value is final
      const float s0 = far[g * D + i];
      sst[idx] = s0;
      if (g >= own_lo && publish) incl_s[(ticket * nkv + g) * D + i] = fmaf(mul, s0, a);
    } else if (g >= own_lo && publish) {
      agg_s[(ticket * nkv + g) * D + i] = a;
    }
  }
  __syncthreads();
  if (tid == 0 && publish) {
    __threadfence();
    for (int g = own_lo; g <= g_hi; ++g) st_release_u32(&flags_s[ticket * nkv + g], first ? kFlagIncl : kFlagAgg);
  }

  // ---- (B) near field: one warp per (token, head), online softmax ---------
  // [P1 §2.1 eq. O_near] over positions max(0, t-k+1) .. t.
  for (int task = warp; task < Tt * p.HPC; task += NW) {
    const int r = task / p.HPC, hh = task % p.HPC;
    const int h = h0 + hh, g = h / G;
    const long long pt = t0 + r;
    float qv[EPL];
    VecLoad<Tin, EPL>::run(qin + ((pt - pos0) * p.nq + h) * D + lane * EPL, qv);
    const long long j0 = (pt - K + 1 > 0) ? pt - K + 1 : 0;
    float m = -INFINITY, den = 0.f, o[EPL];
#pragma unroll
    for (int e = 0; e < EPL; ++e) o[e] = 0.f;
    for (long long j = j0; j <= pt; ++j) {
      const Tin* kp;
      const Tin* vp;
      if (j >= pos0) {
        kp = io.kin + ((j - pos0) * nkv + g) * D;
        vp = io.vin + ((j - pos0) * nkv + g) * D;
      } else {
        const long long off = ((j % K) * nkv + g) * D;
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
#pragma unroll
    for (int e = 0; e < EPL; ++e) xs[r * HS + hh * D + lane * EPL + e] = o[e] * inv;
  }

  // ---- (C) far field: carry-in by decoupled look-back, then the scan -----
  if (!first) {
    for (int gg = 0; gg < NG; ++gg) {
      const int g = g_lo + gg;
      float acc = 0.f, mul = 1.f;
      for (long long j = tile - 1;; --j) {
        const long long u = j * p.n_streams + stream;
        __syncthreads();
        if (tid == 0) s_flag = wait_flag(&flags_s[u * nkv + g], p.spin_limit, p.err);
        __syncthreads();
        const unsigned f = s_flag;
        if (tid < D) {
          const float* src = (f == kFlagIncl ? incl_s : agg_s) + (u * nkv + g) * D;
          acc = fmaf(mul, __ldcg(src + tid), acc);
        }
        if (f == kFlagIncl || j == 0) break;
        mul *= powf(gf, static_cast<float>(evictions(pos0 + j * kTile, kTile)));
      }
      if (tid < D) sst[gg * D + tid] = acc;
    }
    __syncthreads();
    if (publish) {
      const float mul_self = powf(gf, static_cast<float>(evictions(t0, Tt)));
      for (int idx = tid; idx < NG * D; idx += NT) {
        const int g = g_lo + idx / D, i = idx % D;
        if (g >= own_lo) incl_s[(ticket * nkv + g) * D + i] = fmaf(mul_self, sst[idx], sagg[idx]);
      }
      __syncthreads();
      if (tid == 0) {
        __threadfence();
        for (int g = own_lo; g <= g_hi; ++g) st_release_u32(&flags_s[ticket * nkv + g], kFlagIncl);
      }
    }
  }
  __syncthreads();  // near-field O complete in xs; carries in sst
  // Scan: S_t per token, x = O_near + alpha_far * S  [P1 §2.1 eq. O].
  for (int idx = tid; idx < NG * D; idx += NT) {
    const int gg = idx / D, i = idx % D, g = g_lo + gg;
    const int hh_lo = max(0, g * G - h0), hh_hi = min(p.HPC, (g + 1) * G - h0);
    float s = sst[idx];
    for (int r = 0; r < Tt; ++r) {
      const long long pt = t0 + r;
      if (pt >= K) s = ewma(gf, s, to_f32<Tin>(io.key(pt - K, g)[i]));
      for (int hh = hh_lo; hh < hh_hi; ++hh) {
        float* xp = xs + r * HS + hh * D + i;
        *xp = fmaf(p.alpha_far, s, *xp);
      }
    }
    sst[idx] = s;  // S at the end of the tile
  }
  __syncthreads();

  // ---- (D) EMA field aggregate and tail rows for the successor -------------
  if (first) {
    // Carry-in from the state: field, and the 15 ring rows before pos0.
    for (int e = tid; e < HS; e += NT) {
      const int gi = rank * HS + e;
      fcar[e] = field[gi];
      for (int r = 0; r < kHalo; ++r) {
        const long long q = t0 - kHalo + r;
        halo[r * HS + e] = (q >= 0) ? ring[static_cast<size_t>(q % kRing) * p.H + gi] : 0.f;
      }
    }
  }
  {
    const float decay_tile = powf(ge, static_cast<float>(Tt));
    for (int e = tid; e < HS; e += NT) {
      const int gi = rank * HS + e;
      float a = 0.f;
      for (int r = 0; r < Tt; ++r) a = ewma(ge, a, xs[r * HS + e]);
      if (publish) {
        if (first) incl_f[ticket * p.H + gi] = fmaf(decay_tile, fcar[e], a);
        else agg_f[ticket * p.H + gi] = a;
        if (!last)
          for (int r = 0; r < kHalo; ++r)
            halo_ws[(ticket * kHalo + r) * p.H + gi] = xs[(Tt - kHalo + r) * HS + e];
      }
    }
  }
  __syncthreads();
  if (tid == 0 && publish) {
    __threadfence();
    st_release_u32(&flags_f[ticket * p.CS + rank], first ? kFlagIncl : kFlagAgg);
  }

  // ---- (E) pool partial sums over this slice [P3 §2.1 channel 3] ----------
  {
    const float* slot_base = p.slots + static_cast<size_t>(l) * kSlots * p.H + static_cast<size_t>(rank) * HS;
    const int ty = tid / 16, tx = tid % 16;  // rows ty*4..+3, slots tx+16m
    float acc[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[a][c] = 0.f;
    for (int e0 = 0; e0 < HS; e0 += kChunk) {
      __syncthreads();
      for (int idx = tid; idx < kSlots * kChunk; idx += NT) {
        const int j = idx / kChunk, e = idx % kChunk;
        schunk[j * (kChunk + 1) + e] = __ldg(slot_base + static_cast<size_t>(j) * p.H + e0 + e);
      }
      __syncthreads();
#pragma unroll 4
      for (int e = 0; e < kChunk; ++e) {
        float xa[4], sb[4];
#pragma unroll
        for (int a = 0; a < 4; ++a) xa[a] = xs[(ty * 4 + a) * HS + e0 + e];
#pragma unroll
        for (int c = 0; c < 4; ++c) sb[c] = schunk[(tx + 16 * c) * (kChunk + 1) + e];
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
          for (int c = 0; c < 4; ++c) acc[a][c] = fmaf(xa[a], sb[c], acc[a][c]);
      }
    }
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int c = 0; c < 4; ++c) part[(ty * 4 + a) * kPartStride + tx + 16 * c] = acc[a][c];
    for (int r = warp; r < kTile; r += NW) {
      float ss = 0.f;
      for (int e = lane; e < HS; e += 32) ss = fmaf(xs[r * HS + e], xs[r * HS + e], ss);
      ss = warp_sum(ss);
      if (lane == 0) part[r * kPartStride + kSlots] = ss;
    }
  }

  // ---- (F) EMA field carry-in by look-back; predecessor's tail rows -------
  if (!first) {
    for (int e = tid; e < HS; e += NT) fcar[e] = 0.f;
    float mul = 1.f;
    const float decay_full = powf(ge, static_cast<float>(kTile));
    for (long long j = tile - 1;; --j) {
      const long long u = j * p.n_streams + stream;
      __syncthreads();
      if (tid == 0) s_flag = wait_flag(&flags_f[u * p.CS + rank], p.spin_limit, p.err);
      __syncthreads();
      const unsigned f = s_flag;
      const float* src = (f == kFlagIncl ? incl_f : agg_f) + u * p.H + rank * HS;
      for (int e = tid; e < HS; e += NT) fcar[e] = fmaf(mul, __ldcg(src + e), fcar[e]);
      if (j == tile - 1) {
        for (int idx = tid; idx < kHalo * HS; idx += NT) {
          const int r = idx / HS, e = idx % HS;
          halo[idx] = __ldcg(halo_ws + (u * kHalo + r) * p.H + rank * HS + e);
        }
      }
      if (f == kFlagIncl || j == 0) break;
      mul *= decay_full;
    }
    __syncthreads();
    if (publish) {
      const float decay_tile = powf(ge, static_cast<float>(Tt));
      for (int e = tid; e < HS; e += NT) {
        const long long o = ticket * p.H + rank * HS + e;
        incl_f[o] = fmaf(decay_tile, fcar[e], agg_f[o]);
      }
      __syncthreads();
      if (tid == 0) {
        __threadfence();
        st_release_u32(&flags_f[ticket * p.CS + rank], kFlagIncl);
      }
    }
  }

  // ---- (G) cluster reduce-scatter of the pool sums, softmax(cos/T) -------
  cluster.sync();
  {
    const float* nrm = p.slot_norm + static_cast<size_t>(l) * kSlots;
    const float n0 = nrm[lane], n1 = nrm[lane + 32];
    for (int r = rank + p.CS * warp; r < Tt; r += p.CS * NW) {
      float d0 = 0.f, d1 = 0.f, ss = 0.f;
      for (int q = 0; q < p.CS; ++q) {
        const float* rp = cluster.map_shared_rank(part, q) + r * kPartStride;
        d0 += rp[lane];
        d1 += rp[lane + 32];
        ss += rp[kSlots];
      }
      const float nx = fmaxf(sqrtf(ss), kNormFloor);
      const float c0 = d0 / (nx * n0) * p.inv_temp;
      const float c1 = d1 / (nx * n1) * p.inv_temp;
      const float mx = warp_max(fmaxf(c0, c1));
      const float e0 = expf(c0 - mx), e1 = expf(c1 - mx);
      const float inv = 1.f / warp_sum(e0 + e1);
      for (int q = 0; q < p.CS; ++q) {
        float* rw = cluster.map_shared_rank(wts, q) + r * kSlots;
        rw[lane] = e0 * inv;
        rw[lane + 32] = e1 * inv;
      }
    }
  }
  cluster.sync();

  // ---- (H) per element: ring, field, semantic mix, fusion, output ---------
  // [P3 §2.1 channels 1–3, §2.2].
  {
    const float a_l = p.alpha_layer[l];
    const float* slot_col = p.slots + static_cast<size_t>(l) * kSlots * p.H + static_cast<size_t>(rank) * HS;
    float* out = p.out + (in_row0 + (t0 - pos0)) * p.H + rank * HS;
    for (int e = tid; e < HS; e += NT) {
      float sig[kSlots];
#pragma unroll
      for (int j = 0; j < kSlots; ++j) sig[j] = __ldg(slot_col + static_cast<size_t>(j) * p.H + e);
      float rs = 0.f;
#pragma unroll
      for (int r = 0; r < kHalo; ++r) rs += halo[r * HS + e];
      float f = fcar[e];
      for (int r = 0; r < Tt; ++r) {
        const float x = xs[r * HS + e];
        rs += x;
        f = ewma(ge, f, x);
        float sem = 0.f;
        const float* w = wts + r * kSlots;
#pragma unroll
        for (int j = 0; j < kSlots; ++j) sem = fmaf(w[j], sig[j], sem);
        float u = rs * (1.0f / kRing) + 0.5f * f + 0.5f * sem;
        u = fminf(fmaxf(u, -p.clip_eps), p.clip_eps);
        out[static_cast<long long>(r) * p.H + e] = fmaf(a_l, u, x);
        rs -= (r >= kHalo) ? xs[(r - kHalo) * HS + e] : halo[r * HS + e];
      }
      if (last) {
        const int gi = rank * HS + e;
        field[gi] = f;
        // Ring slots of the last 16 positions, and their exact sum.
        const long long t_end = t0 + Tt - 1;
        float tot = 0.f;
        for (int r = 0; r < kRing; ++r) {
          const long long q = t_end - (kRing - 1) + r;
          if (q < 0) continue;
          const long long loc = q - t0;
          const float v = (loc >= 0) ? xs[loc * HS + e] : halo[(loc + kHalo) * HS + e];
          ring[static_cast<size_t>(q % kRing) * p.H + gi] = v;
          tot += v;
        }
        ring_sum[gi] = tot;
      }
    }
  }

  // ---- (I) last tile: window, S and position of the stream ---------------
  if (last) {
    for (int idx = tid; idx < NG * D; idx += NT) {
      const int g = g_lo + idx / D, i = idx % D;
      if (g >= own_lo) far[g * D + i] = sst[idx];
    }
    if (own_lo <= g_hi) {
      const long long t_end = pos0 + p.n - 1;
      const long long w0 = max(pos0, t_end - K + 1);
      const int n_own = g_hi - own_lo + 1;
      const long long cnt = (t_end - w0 + 1) * n_own * D;
      for (long long idx = tid; idx < cnt; idx += NT) {
        const long long j = w0 + idx / (n_own * D);
        const int g = own_lo + static_cast<int>((idx / D) % n_own);
        const int i = static_cast<int>(idx % D);
        const long long src = ((j - pos0) * nkv + g) * D + i;
        const long long dst = ((j % K) * nkv + g) * D + i;
        win_k[dst] = io.kin[src];
        win_v[dst] = io.vin[src];
      }
    }
    if (rank == 0 && tid == 0) *reinterpret_cast<long long*>(blk + p.so.pos) = pos0 + p.n;
  }
}

// Raises the kernel's dynamic shared-memory limit to what the device allows
// (one-time set-up, outside any stream capture).
template <typename Tin, int D>
cudaError_t prepare_t(int optin) {
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, prefill_kernel<Tin, D>);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(prefill_kernel<Tin, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              optin - static_cast<int>(fa.sharedSizeBytes));
}

template <typename Tin, int D>
cudaError_t launch_t(const PrefillParams& p, size_t smem, cudaStream_t s) {
  auto kern = prefill_kernel<Tin, D>;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(p.n_tiles * p.CS), 1, 1);
  cfg.blockDim = dim3(kPrefillThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = p.CS;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, p);
}

}  // namespace

cudaError_t prefill_prepare(int device) {
  int optin = 0;
  cudaError_t e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, device);
  if (e == cudaSuccess) e = prepare_t<float, 64>(optin);
  if (e == cudaSuccess) e = prepare_t<float, 128>(optin);
  if (e == cudaSuccess) e = prepare_t<__nv_bfloat16, 64>(optin);
  if (e == cudaSuccess) e = prepare_t<__nv_bfloat16, 128>(optin);
  return e;
}

size_t prefill_smem_limit(int device) {
  int optin = 0;
  if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, device) != cudaSuccess)
    return 0;
  return static_cast<size_t>(optin) - 1024;  // headroom for the kernel's static shared memory
}

size_t prefill_smem_bytes(int HPC, int head_dim) {
  return static_cast<size_t>(plan_smem(HPC, head_dim).total_floats) * sizeof(float);
}

cudaError_t launch_prefill(const PrefillParams& p, int in_dtype, int head_dim, size_t smem,
                           cudaStream_t s) {
  if (in_dtype == SFA_F32)
    return head_dim == 64 ? launch_t<float, 64>(p, smem, s) : launch_t<float, 128>(p, smem, s);
  return head_dim == 64 ? launch_t<__nv_bfloat16, 64>(p, smem, s)
                        : launch_t<__nv_bfloat16, 128>(p, smem, s);
}

}  // namespace sfa
