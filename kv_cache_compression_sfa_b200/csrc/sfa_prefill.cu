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
// and hence hidden slice [rank*HS, (rank+1)*HS).  Tiles take an ordered
// ticket from a global counter (tile-major over streams), so a tile only
// ever waits on tiles with smaller tickets, which are running or done.
//
// Staging.  The tile's queries and the keys/values it needs (positions
// t0-k .. t0+T-1: the windows plus the keys that leave them) are brought
// into shared memory by the bulk-copy engine in key blocks of up to KB rows;
// the near field runs an online softmax per (token, head) across the blocks
// with the running output kept in the x tile.  The slot slice is staged once
// per tile and feeds both pool contractions.
//
// Recurrences as parallel scans across tiles, with a deterministic
// look-back: tiles are grouped by kGroup; a tile's carry-in is the inclusive
// value at the end of the previous group (or the stream's state) folded with
// the aggregates of the earlier tiles of its own group, always in the same
// order, so results do not depend on timing.
//   * far-field EWMA S (per KV head; depends on keys only) [P1 §2.1 eq. S_t];
//   * EMA field (per hidden element; depends on x) [P3 §2.1 channel 2];
//   * ring mean: a sliding 16-token sum; the 15 rows of x before a tile come
//     from its predecessor's published tail rows (or the state ring).
// Every wait is bounded; a wait that runs out latches SFA_ERR_DEVICE_TIMEOUT
// and the kernel still finishes.
//
// The semantic pool needs |x| and x·slot_j over all of hidden: partial sums
// of the slice are reduce-scattered across the cluster through distributed
// shared memory (rank r finishes tokens r, r+CS, ...) and the softmax
// weights are written into every CTA's shared memory.
#include <cooperative_groups.h>
#include <cuda_bf16.h>

#include <algorithm>

#include "sfa_common.cuh"

namespace cg = cooperative_groups;

namespace sfa {
namespace {

constexpr int NT = kPrefillThreads;
constexpr int NW = NT / 32;
constexpr int kPartStride = kSlots + 1;  // 64 partial dots + |x|^2 per token
constexpr int kCW = 64;                  // columns per combine chunk
constexpr int kSeg = 4;                  // token segments per column in the epilogue
constexpr int kEvChunk = 16;             // evicted-key loads in flight per thread

template <typename Tin, int D>
__global__ void __launch_bounds__(kPrefillThreads, 1)
prefill_kernel(const PrefillParams p) {
  constexpr int EPL = D / 32;
  constexpr int ESZ = static_cast<int>(sizeof(Tin));
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = static_cast<int>(cluster.block_rank());
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  extern __shared__ __align__(16) unsigned char smb[];
  const PrefillPlan& pl = p.plan;
  const int HPC = p.HPC;
  const int HS = HPC * D, XS = HS + 4;
  float* xs = reinterpret_cast<float*>(smb + pl.xs);      // [T][XS]  x (O accumulator first)
  float* halo = reinterpret_cast<float*>(smb + pl.halo);  // [15][HS] x of the 15 tokens before
  float* fcar = reinterpret_cast<float*>(smb + pl.fcar);  // [HS]     field carried in
  float* sst = reinterpret_cast<float*>(smb + pl.sst);    // [NGm][D] S carried in / at tile end
  float* sagg = reinterpret_cast<float*>(smb + pl.sagg);  // [NGm][D] this tile's S aggregate
  float* mrun = reinterpret_cast<float*>(smb + pl.ml);    // [T*HPC]  running max
  float* lrun = mrun + kTile * HPC;                       // [T*HPC]  running denominator
  float* segc = lrun + kTile * HPC;                       // [kSeg][kCW] epilogue carries
  uint64_t* bar_kv = reinterpret_cast<uint64_t*>(smb + pl.bars);
  uint64_t* bar_sl = bar_kv + 1;
  Tin* qst = reinterpret_cast<Tin*>(smb + pl.qst);        // [T][HS]   queries
  unsigned char* kb = smb + pl.kb;                        // [KB][rowB] key block
  unsigned char* vb = smb + pl.vb;                        // [KB][rowB] value block
  float* sl = reinterpret_cast<float*>(smb + pl.sl);      // [64][XS]  slot slice
  float* part = reinterpret_cast<float*>(smb + pl.part);  // [T][65]   pool partials
  float* wts = reinterpret_cast<float*>(smb + pl.wts);    // [T][64]   pool weights
  float* semc = reinterpret_cast<float*>(smb + pl.semc);  // [T][kCW]  semantic chunk

  __shared__ unsigned long long s_ticket;
  __shared__ long long s_pos;
  __shared__ int s_ok;
  __shared__ int s_bad;  // a staging wait ran out: skip global writes

  if (tid == 0) {
    mbar_init(bar_kv, 1);
    mbar_init(bar_sl, 1);
    mbar_fence_init();
    s_bad = 0;
  }
  pdl_trigger();
  pdl_wait();

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
  const bool last = (tile == p.tiles_per_stream - 1);
  const bool publish = (ticket != p.withhold_tile);
  const long long gstart = (tile / kGroup) * kGroup;         // first tile of this group
  const bool group_end = (tile % kGroup == kGroup - 1) && !last;

  unsigned char* blk = p.state + kHeaderBytes + static_cast<long long>(stream) * p.so.stride;
  if (tid == 0) s_pos = *reinterpret_cast<const volatile long long*>(blk + p.so.pos);
  __syncthreads();
  const long long pos0 = s_pos;
  Tin* win_k = reinterpret_cast<Tin*>(blk + p.so.win_k);
  Tin* win_v = reinterpret_cast<Tin*>(blk + p.so.win_v);
  float* far = reinterpret_cast<float*>(blk + p.so.far);
  float* field = reinterpret_cast<float*>(blk + p.so.field);
  float* ring_sum = reinterpret_cast<float*>(blk + p.so.ring_sum);
  float* ring = reinterpret_cast<float*>(blk + p.so.ring);

  const long long t0 = pos0 + tile * kTile;  // first position of the tile
  const int Tt = static_cast<int>(min(static_cast<long long>(kTile), p.n - tile * kTile));
  const int K = p.K, G = p.G, nkv = p.nkv;
  const int h0 = rank * HPC;
  const int g_lo = h0 / G, g_hi = (h0 + HPC - 1) / G;
  const int NG = g_hi - g_lo + 1;
  const int own_lo = (h0 + G - 1) / G;  // KV heads whose carries this CTA publishes
  const float gf = p.gamma_far, ge = p.ema_gamma;
  const int rowB = p.NGm * D * ESZ + 16;  // padded key/value row in shared memory

  const long long in_row0 = static_cast<long long>(stream) * p.n;  // first input row of the stream
  const Tin* kin = static_cast<const Tin*>(p.k) + in_row0 * nkv * D;
  const Tin* vin = static_cast<const Tin*>(p.v) + in_row0 * nkv * D;
  const Tin* qin = static_cast<const Tin*>(p.q) + in_row0 * p.nq * D;

  unsigned* fs_agg = reinterpret_cast<unsigned*>(p.ws + p.ws_fs_agg);
  unsigned* fs_incl = reinterpret_cast<unsigned*>(p.ws + p.ws_fs_incl);
  unsigned* ff_agg = reinterpret_cast<unsigned*>(p.ws + p.ws_ff_agg);
  unsigned* ff_incl = reinterpret_cast<unsigned*>(p.ws + p.ws_ff_incl);
  float* agg_s = reinterpret_cast<float*>(p.ws + p.ws_agg_s);
  float* incl_s = reinterpret_cast<float*>(p.ws + p.ws_incl_s);
  float* agg_f = reinterpret_cast<float*>(p.ws + p.ws_agg_f);
  float* incl_f = reinterpret_cast<float*>(p.ws + p.ws_incl_f);
  float* halo_ws = reinterpret_cast<float*>(p.ws + p.ws_halo);

  // Key row of absolute position j >= 0 for KV head g: from the input if it
  // belongs to this call, else from window slot j mod k (the state holds
  // positions pos0-k .. pos0-1).
  auto key_row = [&](long long j, int g) -> const Tin* {
    return (j >= pos0) ? kin + ((j - pos0) * nkv + g) * D : win_k + ((j % K) * nkv + g) * D;
  };
  auto evictions = [&](long long a, int len) -> int {  // positions p in [a, a+len) with p >= k
    const long long lo = a > K ? a : static_cast<long long>(K);
    const long long hi = a + len;
    return hi > lo ? static_cast<int>(hi - lo) : 0;
  };
  auto ticket_of = [&](long long j) -> long long { return j * p.n_streams + stream; };

  // ---- staging of block `bi` of key/value rows (and the queries with block 0)
  const long long kv_start = t0 - K;                       // position of block row 0
  const int kv_rows = Tt + K;                              // positions t0-k .. t0+Tt-1
  const int n_blocks = (kv_rows + p.KB - 1) / p.KB;
  auto issue_block = [&](int bi) {
    if (warp != 0) return;
    const long long bs = kv_start + static_cast<long long>(bi) * p.KB;
    const int rows = min(p.KB, kv_rows - bi * p.KB);
    const long long first_valid = bs < 0 ? -bs : 0;      // rows at negative positions stay unused
    const int valid = rows > first_valid ? rows - static_cast<int>(first_valid) : 0;
    const unsigned row_bytes = static_cast<unsigned>(NG * D * ESZ);
    unsigned bytes = 2u * row_bytes * valid;
    if (bi == 0) bytes += static_cast<unsigned>(Tt * HS * ESZ);
    fence_proxy_async_smem();
    if (lane == 0) mbar_arrive_expect_tx(bar_kv, bytes);
    __syncwarp();
    for (int r = static_cast<int>(first_valid) + lane; r < rows; r += 32) {
      const long long j = bs + r;
      const Tin* ks = (j >= pos0) ? kin + ((j - pos0) * nkv + g_lo) * D : win_k + ((j % K) * nkv + g_lo) * D;
      const Tin* vs = (j >= pos0) ? vin + ((j - pos0) * nkv + g_lo) * D : win_v + ((j % K) * nkv + g_lo) * D;
      bulk_g2s(kb + r * rowB, ks, row_bytes, bar_kv);
      bulk_g2s(vb + r * rowB, vs, row_bytes, bar_kv);
    }
    if (bi == 0)
      for (int r = lane; r < Tt; r += 32)
        bulk_g2s(qst + r * HS, qin + ((t0 - pos0 + r) * p.nq + h0) * D,
                 static_cast<unsigned>(HS * ESZ), bar_kv);
  };
  issue_block(0);

  // ---- (A) far field: this tile's aggregate of the keys leaving the window
  // (read straight from global memory, independent loads in flight).
  for (int idx = tid; idx < NG * D; idx += NT) {
    const int gg = idx / D, i = idx % D, g = g_lo + gg;
    float a = 0.f;
    for (int r0 = 0; r0 < Tt; r0 += kEvChunk) {
      float ev[kEvChunk];
#pragma unroll
      for (int u = 0; u < kEvChunk; ++u) {
        const long long pt = t0 + r0 + u;
        ev[u] = (r0 + u < Tt && pt >= K) ? to_f32<Tin>(key_row(pt - K, g)[i]) : 0.f;
      }
#pragma unroll
      for (int u = 0; u < kEvChunk; ++u)
        if (r0 + u < Tt && t0 + r0 + u >= K) a = ewma(gf, a, ev[u]);
    }
    sagg[idx] = a;
    if (g >= own_lo && publish) agg_s[(ticket * nkv + g) * D + i] = a;
  }
  // running state of the near field
  for (int i = tid; i < kTile * HPC; i += NT) {
    mrun[i] = -INFINITY;
    lrun[i] = 0.f;
  }
  for (int i = tid; i < kTile * XS; i += NT) xs[i] = 0.f;
  __syncthreads();
  if (tid == 0 && publish) {
    __threadfence();
    for (int g = own_lo; g <= g_hi; ++g) st_release_u32(&fs_agg[ticket * nkv + g], 1u);
  }

  // ---- (B) near field [P1 §2.1 eq. O_near]: per key block, each warp takes
  // (token, head) pairs; lane a scores key cb+a in full, online softmax,
  // then P·V with lanes over head dims into the x tile.
  for (int bi = 0; bi < n_blocks; ++bi) {
    if (!mbar_wait_bounded(bar_kv, bi & 1, kMbarPollLimit, p.err)) s_bad = 1;
    const long long bs = kv_start + static_cast<long long>(bi) * p.KB;
    const long long be = bs + min(p.KB, kv_rows - bi * p.KB);  // exclusive
    for (int pair = warp; pair < Tt * HPC; pair += NW) {
      const int r = pair / HPC, hh = pair % HPC;
      const int gg = (h0 + hh) / G - g_lo;
      const long long pt = t0 + r;
      const long long wlo = pt - K + 1 > 0 ? pt - K + 1 : 0;
      const long long lo = wlo > bs ? wlo : bs;
      const long long hi = pt < be - 1 ? pt : be - 1;
      if (lo > hi) continue;
      const Tin* qrow = qst + r * HS + hh * D;
      float* orow = xs + r * XS + hh * D + lane * EPL;
      float m = mrun[pair], den = lrun[pair];
      float o[EPL];
#pragma unroll
      for (int e = 0; e < EPL; ++e) o[e] = orow[e];
      for (long long cb = lo; cb <= hi; cb += 32) {
        const int cnt = static_cast<int>(min(32LL, hi - cb + 1));
        float s = -INFINITY;
        if (lane < cnt) {
          const Tin* kr = reinterpret_cast<const Tin*>(kb + (cb + lane - bs) * rowB) + gg * D;
          constexpr int VE = Load16<Tin>::N;
          float acc = 0.f;
#pragma unroll
          for (int i = 0; i < D; i += VE) {
            float kv[VE], qv[VE];
            Load16<Tin>::run(kr + i, kv);
            Load16<Tin>::run(qrow + i, qv);
#pragma unroll
            for (int e = 0; e < VE; ++e) acc = fmaf(qv[e], kv[e], acc);
          }
          s = acc * p.score_scale;
        }
        const float mn = fmaxf(m, warp_max(s));
        const float corr = expf(m - mn);
        const float pj = (lane < cnt) ? expf(s - mn) : 0.f;
        den = fmaf(den, corr, warp_sum(pj));
#pragma unroll
        for (int e = 0; e < EPL; ++e) o[e] *= corr;
        for (int c = 0; c < cnt; ++c) {
          const float pc = __shfl_sync(0xffffffffu, pj, c);
          const Tin* vr = reinterpret_cast<const Tin*>(vb + (cb + c - bs) * rowB) + gg * D + lane * EPL;
          float vv[EPL];
          VecLoad<Tin, EPL>::run(vr, vv);
#pragma unroll
          for (int e = 0; e < EPL; ++e) o[e] = fmaf(pc, vv[e], o[e]);
        }
        m = mn;
      }
#pragma unroll
      for (int e = 0; e < EPL; ++e) orow[e] = o[e];
      if (lane == 0) {
        mrun[pair] = m;
        lrun[pair] = den;
      }
    }
    __syncthreads();  // the block buffers are free again
    if (bi + 1 < n_blocks) issue_block(bi + 1);
  }
  // normalise: O = acc / den
  for (int idx = tid; idx < Tt * HS; idx += NT) {
    const int r = idx / HS, c = idx % HS;
    xs[r * XS + c] /= lrun[r * HPC + c / D];
  }

  // Slot slice for both pool contractions; the staging buffers are free.
  const float* slot_base = p.slots + static_cast<size_t>(l) * kSlots * p.H + static_cast<size_t>(rank) * HS;
  if (warp == 0) {
    fence_proxy_async_smem();
    if (lane == 0) mbar_arrive_expect_tx(bar_sl, kSlots * HS * 4u);
    __syncwarp();
    for (int j = lane; j < kSlots; j += 32)
      bulk_g2s(sl + j * XS, slot_base + static_cast<size_t>(j) * p.H, HS * 4u, bar_sl);
  }

  // ---- (C) far field carry-in (deterministic look-back), then the scan --
  // carry = INCL(end of previous group) or the state, folded with the
  // aggregates of the group's earlier tiles in order.
  {
    const bool from_state = (gstart == 0);
    if (!from_state) {
      if (tid == 0)
        for (int g = g_lo; g <= g_hi; ++g) wait_flag(&fs_incl[ticket_of(gstart - 1) * nkv + g], p.spin_limit, p.err);
      __syncthreads();
    }
    for (int idx = tid; idx < NG * D; idx += NT) {
      const int g = g_lo + idx / D, i = idx % D;
      sst[idx] = from_state ? far[g * D + i] : __ldcg(incl_s + (ticket_of(gstart - 1) * nkv + g) * D + i);
    }
    for (long long j = gstart; j < tile; ++j) {
      __syncthreads();
      if (tid == 0)
        for (int g = g_lo; g <= g_hi; ++g) wait_flag(&fs_agg[ticket_of(j) * nkv + g], p.spin_limit, p.err);
      __syncthreads();
      const float mul = powf(gf, static_cast<float>(evictions(pos0 + j * kTile, kTile)));
      for (int idx = tid; idx < NG * D; idx += NT) {
        const int g = g_lo + idx / D, i = idx % D;
        sst[idx] = fmaf(mul, sst[idx], __ldcg(agg_s + (ticket_of(j) * nkv + g) * D + i));
      }
    }
    __syncthreads();
    if (group_end && publish) {
      const float mul = powf(gf, static_cast<float>(evictions(t0, Tt)));
      for (int idx = tid; idx < NG * D; idx += NT) {
        const int g = g_lo + idx / D, i = idx % D;
        if (g >= own_lo) incl_s[(ticket * nkv + g) * D + i] = fmaf(mul, sst[idx], sagg[idx]);
      }
      __syncthreads();
      if (tid == 0) {
        __threadfence();
        for (int g = own_lo; g <= g_hi; ++g) st_release_u32(&fs_incl[ticket * nkv + g], 1u);
      }
    }
  }
  // scan: S_t per token, x = O_near + alpha_far * S_t  [P1 §2.1 eq. O]
  for (int idx = tid; idx < NG * D; idx += NT) {
    const int gg = idx / D, i = idx % D, g = g_lo + gg;
    const int hh_lo = max(0, g * G - h0), hh_hi = min(HPC, (g + 1) * G - h0);
    float s = sst[idx];
    for (int r0 = 0; r0 < Tt; r0 += kEvChunk) {
      float ev[kEvChunk];
#pragma unroll
      for (int u = 0; u < kEvChunk; ++u) {
        const long long pt = t0 + r0 + u;
        ev[u] = (r0 + u < Tt && pt >= K) ? to_f32<Tin>(key_row(pt - K, g)[i]) : 0.f;
      }
#pragma unroll
      for (int u = 0; u < kEvChunk; ++u) {
        const int r = r0 + u;
        if (r < Tt) {
          if (t0 + r >= K) s = ewma(gf, s, ev[u]);
          for (int hh = hh_lo; hh < hh_hi; ++hh) {
            float* xp = xs + r * XS + hh * D + i;
            *xp = fmaf(p.alpha_far, s, *xp);
          }
        }
      }
    }
    sst[idx] = s;  // S at the end of the tile
  }
  __syncthreads();

  // ---- (D) EMA field aggregate; tail rows for the successor -------------
  // Tiles of the first group read the state field (and tile 0 the state
  // ring rows) now, before any flag is published: the stream's last tile
  // overwrites them once every earlier tile has published.
  if (gstart == 0)
    for (int e = tid; e < HS; e += NT) fcar[e] = field[rank * HS + e];
  if (tile == 0)
    for (int idx = tid; idx < kHalo * HS; idx += NT) {
      const int r = idx / HS, e = idx % HS;
      const long long q = t0 - kHalo + r;
      halo[idx] = (q >= 0) ? ring[static_cast<size_t>(q % kRing) * p.H + rank * HS + e] : 0.f;
    }
  for (int e = tid; e < HS; e += NT) {
    float a = 0.f;
    for (int r = 0; r < Tt; ++r) a = ewma(ge, a, xs[r * XS + e]);
    if (publish) {
      agg_f[ticket * p.H + rank * HS + e] = a;
      if (!last)
        for (int r = 0; r < kHalo; ++r)
          halo_ws[(ticket * kHalo + r) * p.H + rank * HS + e] = xs[(Tt - kHalo + r) * XS + e];
    }
  }
  __syncthreads();
  if (tid == 0 && publish) {
    __threadfence();
    st_release_u32(&ff_agg[ticket * p.CS + rank], 1u);
  }

  // ---- (E) pool partial sums over this slice [P3 §2.1 channel 3] ---------
  // scores[T x 64] = x[T x HS] · slot^T, register-blocked 4 tokens x 4 slots.
  if (!mbar_wait_bounded(bar_sl, 0, kMbarPollLimit, p.err)) s_bad = 1;
  {
    const int ty = tid / 16, tx = tid % 16;
    float acc[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[a][c] = 0.f;
    for (int e = 0; e < HS; e += 4) {
      float4 xa[4], sb[4];
#pragma unroll
      for (int a = 0; a < 4; ++a) xa[a] = *reinterpret_cast<const float4*>(xs + (ty * 4 + a) * XS + e);
#pragma unroll
      for (int c = 0; c < 4; ++c) sb[c] = *reinterpret_cast<const float4*>(sl + (tx + 16 * c) * XS + e);
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int c = 0; c < 4; ++c)
          acc[a][c] = fmaf(xa[a].x, sb[c].x, fmaf(xa[a].y, sb[c].y,
                      fmaf(xa[a].z, sb[c].z, fmaf(xa[a].w, sb[c].w, acc[a][c]))));
    }
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int c = 0; c < 4; ++c) part[(ty * 4 + a) * kPartStride + tx + 16 * c] = acc[a][c];
    for (int r = warp; r < kTile; r += NW) {
      float ss = 0.f;
      for (int e = lane; e < HS; e += 32) ss = fmaf(xs[r * XS + e], xs[r * XS + e], ss);
      ss = warp_sum(ss);
      if (lane == 0) part[r * kPartStride + kSlots] = ss;
    }
  }

  // ---- (F) EMA field carry-in (deterministic look-back); tail rows ------
  {
    if (gstart > 0) {
      if (tid == 0) wait_flag(&ff_incl[ticket_of(gstart - 1) * p.CS + rank], p.spin_limit, p.err);
      __syncthreads();
      for (int e = tid; e < HS; e += NT)
        fcar[e] = __ldcg(incl_f + ticket_of(gstart - 1) * p.H + rank * HS + e);
    }
    const float mul_full = powf(ge, static_cast<float>(kTile));
    for (long long j = gstart; j < tile; ++j) {
      __syncthreads();
      if (tid == 0) wait_flag(&ff_agg[ticket_of(j) * p.CS + rank], p.spin_limit, p.err);
      __syncthreads();
      for (int e = tid; e < HS; e += NT)
        fcar[e] = fmaf(mul_full, fcar[e], __ldcg(agg_f + ticket_of(j) * p.H + rank * HS + e));
    }
    if (tile > 0) {  // x rows of the 15 tokens before the tile, from the predecessor
      if (tid == 0) wait_flag(&ff_agg[ticket_of(tile - 1) * p.CS + rank], p.spin_limit, p.err);
      __syncthreads();
      for (int idx = tid; idx < kHalo * HS; idx += NT) {
        const int r = idx / HS, e = idx % HS;
        halo[idx] = __ldcg(halo_ws + (ticket_of(tile - 1) * kHalo + r) * p.H + rank * HS + e);
      }
    }
    __syncthreads();
    if (group_end && publish) {
      const float mul = powf(ge, static_cast<float>(Tt));
      for (int e = tid; e < HS; e += NT) {
        const long long o = ticket * p.H + rank * HS + e;
        incl_f[o] = fmaf(mul, fcar[e], agg_f[o]);
      }
      __syncthreads();
      if (tid == 0) {
        __threadfence();
        st_release_u32(&ff_incl[ticket * p.CS + rank], 1u);
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

  // ---- (H) per column chunk: semantic mix (GEMM), then ring, field,
  // fusion, clip, output [P3 §2.1 channels 1–3, §2.2].
  const float a_l = p.alpha_layer[l];
  const bool write_ok = !s_bad;
  float* out = p.out + (in_row0 + (t0 - pos0)) * p.H + rank * HS;
  for (int c0 = 0; c0 < HS; c0 += kCW) {
    {  // semc[T x 64] = wts[T x 64] · slot[64 x cols c0..c0+63]
      const int ty = tid / 16, tx = tid % 16;
      float acc[4][4];
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[a][c] = 0.f;
#pragma unroll 4
      for (int j = 0; j < kSlots; ++j) {
        const float4 s4 = *reinterpret_cast<const float4*>(sl + j * XS + c0 + tx * 4);
#pragma unroll
        for (int a = 0; a < 4; ++a) {
          const float w = wts[(ty * 4 + a) * kSlots + j];
          acc[a][0] = fmaf(w, s4.x, acc[a][0]);
          acc[a][1] = fmaf(w, s4.y, acc[a][1]);
          acc[a][2] = fmaf(w, s4.z, acc[a][2]);
          acc[a][3] = fmaf(w, s4.w, acc[a][3]);
        }
      }
#pragma unroll
      for (int a = 0; a < 4; ++a)
        *reinterpret_cast<float4*>(semc + (ty * 4 + a) * kCW + tx * 4) =
            make_float4(acc[a][0], acc[a][1], acc[a][2], acc[a][3]);
    }
    // field: per-segment aggregates, then carries folded in segment order
    const int c = tid % kCW, sg = tid / kCW;  // column, token segment
    const int e = c0 + c;
    const int r_lo = sg * (kTile / kSeg), r_hi = min(Tt, r_lo + kTile / kSeg);
    {
      float a = 0.f;
      for (int r = r_lo; r < r_hi; ++r) a = ewma(ge, a, xs[r * XS + e]);
      segc[sg * kCW + c] = a;
    }
    __syncthreads();
    float f = fcar[e];
    for (int s2 = 0; s2 < sg; ++s2) {
      const int len = max(0, min(Tt, (s2 + 1) * (kTile / kSeg)) - s2 * (kTile / kSeg));
      f = fmaf(powf(ge, static_cast<float>(len)), f, segc[s2 * kCW + c]);
    }
    // ring: sum of the 16 positions ending at r, from the x tile and the halo
    auto xat = [&](int r) -> float { return r >= 0 ? xs[r * XS + e] : halo[(r + kHalo) * HS + e]; };
    float rs = 0.f;
    if (r_lo < r_hi)
      for (int r = r_lo - kHalo; r <= r_lo; ++r) rs += xat(r);
    for (int r = r_lo; r < r_hi; ++r) {
      if (r > r_lo) rs += xat(r) - xat(r - kRing);
      const float x = xs[r * XS + e];
      f = ewma(ge, f, x);
      float u = rs * (1.0f / kRing) + 0.5f * f + 0.5f * semc[r * kCW + c];
      u = fminf(fmaxf(u, -p.clip_eps), p.clip_eps);
      if (write_ok) out[static_cast<long long>(r) * p.H + e] = fmaf(a_l, u, x);
    }
    if (last && write_ok) {
      const int gi = rank * HS + e;
      if (r_lo < Tt && r_hi == Tt) field[gi] = f;  // the segment holding the last token
      if (sg == 0) {
        // ring slots of the last 16 positions, and their exact sum
        const long long t_end = t0 + Tt - 1;
        float tot = 0.f;
        for (int r = 0; r < kRing; ++r) {
          const long long q = t_end - (kRing - 1) + r;
          if (q < 0) continue;
          const float v = xat(static_cast<int>(q - t0));
          ring[static_cast<size_t>(q % kRing) * p.H + gi] = v;
          tot += v;
        }
        ring_sum[gi] = tot;
      }
    }
    __syncthreads();
  }

  // ---- (I) last tile: window, S and position of the stream ---------------
  if (last && write_ok) {
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
        win_k[dst] = kin[src];
        win_v[dst] = vin[src];
      }
    }
    if (rank == 0 && tid == 0) *reinterpret_cast<long long*>(blk + p.so.pos) = pos0 + p.n;
  }
}

template <typename Tin, int D>
cudaError_t prepare_t(int optin) {
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, prefill_kernel<Tin, D>);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(prefill_kernel<Tin, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             optin - static_cast<int>(fa.sharedSizeBytes));
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(prefill_kernel<Tin, D>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  return e;
}

template <typename Tin, int D>
cudaError_t launch_t(const PrefillParams& p, cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(p.n_tiles * p.CS), 1, 1);
  cfg.blockDim = dim3(kPrefillThreads, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(p.plan.total);
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
  return cudaLaunchKernelEx(&cfg, prefill_kernel<Tin, D>, p);
}

}  // namespace

// Shared-memory plan: persistent regions, then a union of the staging
// buffers (near-field phase) and the pool buffers (pool phase).  The key
// block is as tall as fits, up to the whole span t0-k .. t0+T-1.
bool plan_prefill(int HPC, int D, int esz, int NGm, int K, size_t budget, PrefillPlan* out) {
  const int HS = HPC * D, XS = HS + 4;
  auto a16 = [](long long x) { return static_cast<int>((x + 15) & ~15LL); };
  PrefillPlan p;
  int off = 0;
  p.bars = off;                 off += 16;
  p.xs = off;                   off += a16(4LL * kTile * XS);
  p.halo = off;                 off += a16(4LL * kHalo * HS);
  p.fcar = off;                 off += a16(4LL * HS);
  p.sst = off;                  off += a16(4LL * NGm * D);
  p.sagg = off;                 off += a16(4LL * NGm * D);
  p.ml = off;                   off += a16(4LL * (2 * kTile * HPC + kSeg * kCW));
  p.u0 = off;
  // pool phase
  int q = off;
  p.sl = q;                     q += a16(4LL * kSlots * XS);
  p.part = q;                   q += a16(4LL * kTile * kPartStride);
  p.wts = q;                    q += a16(4LL * kTile * kSlots);
  p.semc = q;                   q += a16(4LL * kTile * kCW);
  const int pool_end = q;
  // staging phase
  q = off;
  p.qst = q;                    q += a16(static_cast<long long>(kTile) * HS * esz);
  const int row_b = NGm * D * esz + 16;
  const long long room = static_cast<long long>(budget) - q;
  int kb_rows = static_cast<int>(room / (2LL * row_b));
  kb_rows = std::min(kb_rows, kTile + K);
  if (kb_rows < 32) return false;
  p.KB = kb_rows;
  p.kb = q;                     q += a16(static_cast<long long>(row_b) * kb_rows);
  p.vb = q;                     q += a16(static_cast<long long>(row_b) * kb_rows);
  p.total = std::max(q, pool_end);
  if (static_cast<size_t>(p.total) > budget) return false;
  *out = p;
  return true;
}

template <typename Tin, int D>
int max_clusters_t(int cs, size_t smem) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(cs * 16), 1, 1);
  cfg.blockDim = dim3(kPrefillThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cs;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, prefill_kernel<Tin, D>, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return n;
}

int prefill_max_active_clusters(int cs, size_t smem, int in_dtype, int head_dim) {
  if (in_dtype == SFA_F32) return head_dim == 64 ? max_clusters_t<float, 64>(cs, smem) : max_clusters_t<float, 128>(cs, smem);
  return head_dim == 64 ? max_clusters_t<__nv_bfloat16, 64>(cs, smem)
                        : max_clusters_t<__nv_bfloat16, 128>(cs, smem);
}

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

cudaError_t launch_prefill(const PrefillParams& p, int in_dtype, int head_dim, cudaStream_t s) {
  if (in_dtype == SFA_F32) return head_dim == 64 ? launch_t<float, 64>(p, s) : launch_t<float, 128>(p, s);
  return head_dim == 64 ? launch_t<__nv_bfloat16, 64>(p, s) : launch_t<__nv_bfloat16, 128>(p, s);
}

}  // namespace sfa
