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
// with the running output kept in the x tile (two (token, head) pairs per
// warp when k <= 16).
//
// Semantic pool on the tensor cores (tcgen05, accumulators in tensor
// memory): scores[T x 64] = x[T x HS] . slot^T and sem[T x HS] =
// w[T x 64] . slot, each as three bf16 MMAs (hi*hi + hi*lo + lo*hi of the
// split operands, about 16 significant bits) accumulated in fp32.  The slot
// slice arrives by bulk copy as bf16 hi/lo blocks laid out at sfa_init so
// that one copy feeds both contractions.
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
// The pool needs |x| and x·slot_j over all of hidden: partial sums of the
// slice are reduce-scattered across the cluster through distributed shared
// memory (rank r finishes tokens r, r+CS, ...) and the softmax weights are
// written into every CTA's shared memory.
#include <cooperative_groups.h>
#include <cstring>
#include <type_traits>
#include <cuda_bf16.h>

#include <algorithm>

#include "sfa_common.cuh"
#include "sfa_umma.cuh"

namespace cg = cooperative_groups;

namespace sfa {
namespace {

constexpr int NT = kPrefillThreads;
constexpr int NW = NT / 32;
constexpr int kPartStride = kSlots + 1;  // 64 partial dots + |x|^2 per token
constexpr int kCW = kBlk;                // columns per combine chunk
constexpr int kSemStride = kCW + 4;      // padded row of the sem chunk
constexpr int kSeg = 4;                  // token segments per column in the epilogue
constexpr int kEvChunk = 16;             // evicted-key loads in flight per thread
constexpr int kTmemCols = 256;           // scores (64) + two 64-column sem buffers
// Tensor-core near field: key span t0-16 .. t0+63 of a tile (k <= 16) as the
// N of the score MMA, 8-row groups of that span, and the column of the
// P·V accumulator in tensor memory.
constexpr int kSpan = kTile + 16;
constexpr int kSpanR8 = kSpan / 8;
constexpr int kTmemO = 128;
static_assert(kTile == kBlk, "tile tokens are the M of the pool MMAs");

// Near field over one staged key block for all (token, head) pairs of the
// tile [P1 §2.1 eq. O_near].  LP lanes serve one pair: lane a scores key
// lo+base+a in full, online softmax across chunks and blocks, then P·V with
// the LP lanes over head dims, accumulated into the pair's row of the x
// tile.  Running max and denominator per pair live in mrun/lrun.
template <typename Tin, int D, int LP>
__device__ __forceinline__ void near_block(const Tin* qst, const unsigned char* kb,
                                           const unsigned char* vb, float* xs, float* mrun,
                                           float* lrun, int rowB, int HS, int XS, int HPC, int G,
                                           int g_lo, int K, long long t0, int Tt, long long bs,
                                           long long be, float score_scale, int h0, int warp,
                                           int lane) {
  constexpr int PPW = 32 / LP;  // pairs per warp
  constexpr int EPL = D / LP;   // head dims per lane in P·V
  constexpr int VE = Load16<Tin>::N;
  const int sub = lane / LP, sl = lane % LP;
  const int gbase = sub * LP;   // first lane of this sub-group
  for (int pb = warp * PPW; pb < Tt * HPC; pb += NW * PPW) {
    const int pair = pb + sub;
    const bool live = pair < Tt * HPC;
    const int r = live ? pair / HPC : 0;
    const int hh = live ? pair % HPC : 0;
    const int gg = (h0 + hh) / G - g_lo;  // KV head of this pair, local to the CTA
    const long long pt = t0 + r;
    const long long wlo = pt - K + 1 > 0 ? pt - K + 1 : 0;
    const long long lo = wlo > bs ? wlo : bs;
    const long long hi = pt < be - 1 ? pt : be - 1;
    const int cnt_pair = (live && lo <= hi) ? static_cast<int>(hi - lo + 1) : 0;
    int cnt_max = cnt_pair;  // the sub-pairs of a warp run the same number of chunks
    if (LP < 32) cnt_max = max(cnt_max, __shfl_xor_sync(0xffffffffu, cnt_max, 16));
    if (cnt_max == 0) continue;
    float* orow = xs + r * XS + hh * D + sl * EPL;
    float m = live ? mrun[pair] : 0.f;
    float den = live ? lrun[pair] : 0.f;
    float o[EPL];
#pragma unroll
    for (int e = 0; e < EPL; ++e) o[e] = live ? orow[e] : 0.f;
    const Tin* qrow = qst + r * HS + hh * D;
    for (int base = 0; base < cnt_max; base += LP) {
      const int cnt = max(0, min(LP, cnt_pair - base));
      float s = -INFINITY;
      if (sl < cnt) {
        const Tin* kr = reinterpret_cast<const Tin*>(kb + (lo + base + sl - bs) * rowB) + gg * D;
        float acc[4] = {0.f, 0.f, 0.f, 0.f};  // independent chains
#pragma unroll
        for (int i = 0; i < D; i += VE) {
          float kv[VE], qv[VE];
          Load16<Tin>::run(kr + i, kv);
          Load16<Tin>::run(qrow + i, qv);
#pragma unroll
          for (int e = 0; e < VE; ++e) acc[e & 3] = fmaf(qv[e], kv[e], acc[e & 3]);
        }
        s = ((acc[0] + acc[1]) + (acc[2] + acc[3])) * score_scale;
      }
      float cm = s;
#pragma unroll
      for (int off = LP / 2; off > 0; off >>= 1) cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, off));
      const float mn = (cnt > 0) ? fmaxf(m, cm) : m;
      const float corr = (cnt > 0) ? expf(m - mn) : 1.f;
      const float pj = (sl < cnt) ? expf(s - mn) : 0.f;
      float ps = pj;
#pragma unroll
      for (int off = LP / 2; off > 0; off >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
      den = fmaf(den, corr, ps);
#pragma unroll
      for (int e = 0; e < EPL; ++e) o[e] *= corr;
      const int cmax = min(LP, cnt_max - base);
      for (int c = 0; c < cmax; ++c) {
        const float pc = __shfl_sync(0xffffffffu, pj, gbase + c);
        if (c < cnt) {
          const Tin* vr = reinterpret_cast<const Tin*>(vb + (lo + base + c - bs) * rowB) + gg * D + sl * EPL;
          float vv[EPL];
          VecLoad<Tin, EPL>::run(vr, vv);
#pragma unroll
          for (int e = 0; e < EPL; ++e) o[e] = fmaf(pc, vv[e], o[e]);
        }
      }
      m = mn;
    }
    if (live) {
#pragma unroll
      for (int e = 0; e < EPL; ++e) orow[e] = o[e];
      if (sl == 0) {
        mrun[pair] = m;
        lrun[pair] = den;
      }
    }
  }
}

template <typename Tin, int D>
__global__ void __launch_bounds__(kPrefillThreads, 2)
prefill_kernel(const PrefillParams p) {
  constexpr int ESZ = static_cast<int>(sizeof(Tin));
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = static_cast<int>(cluster.block_rank());
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  extern __shared__ __align__(16) unsigned char smb[];
  const PrefillPlan& pl = p.plan;
  const int HPC = p.HPC;
  const int HS = HPC * D, XS = HS + 4;
  const int nch = HS / kBlk;                               // 64-column chunks of the slice
  uint64_t* bars = reinterpret_cast<uint64_t*>(smb + pl.bars);
  uint64_t* bar_kv = bars + 0;                             // key/value blocks (+ queries)
  uint64_t* bar_sl = bars + 1;                             // slot image
  uint64_t* bar_ms = bars + 2;                             // [2] score MMAs done, per x buffer
  uint64_t* bar_sd = bars + 4;                             // all score MMAs done
  uint64_t* bar_mc = bars + 5;                             // [2] sem MMAs done, per accumulator
  uint64_t* bar_nf = bars + 7;                             // near-field MMAs done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 8);
  float* xs = reinterpret_cast<float*>(smb + pl.xs);      // [T][XS]  x (O accumulator first)
  float* halo = reinterpret_cast<float*>(smb + pl.halo);  // [15][HS] x of the 15 tokens before
  float* fcar = reinterpret_cast<float*>(smb + pl.fcar);  // [HS]     field carried in
  float* sst = reinterpret_cast<float*>(smb + pl.sst);    // [NGm][D] S carried in / at tile end
  float* sagg = reinterpret_cast<float*>(smb + pl.sagg);  // [NGm][D] this tile's S aggregate
  float* segA = reinterpret_cast<float*>(smb + pl.sega);  // [nseg][NG*D] scan segment aggregates
  float* segc = reinterpret_cast<float*>(smb + pl.ml);    // [kSeg][kCW] epilogue carries
  float* mrun = segc + kSeg * kCW;                        // [T*HPC]  running max (CUDA-core near field)
  float* lrun = mrun + kTile * HPC;                       // [T*HPC]  running denominator
  Tin* qst = reinterpret_cast<Tin*>(smb + pl.qst);        // [T][HS]   queries
  unsigned char* kb = smb + pl.kb;                        // [KB][rowB] key block
  unsigned char* vb = smb + pl.vb;                        // [KB][rowB] value block
  // tensor-core near field: packed query block [64 x D], key and value blocks
  // [kSpan x D] per KV head, P block [64 x kSpan] (hi, lo)
  unsigned char* qa = smb + pl.qa;
  unsigned char* kvp = smb + pl.kvp;
  unsigned char* pa = smb + pl.pa;
  const bool tc = pl.tc != 0;
  unsigned char* simg = smb + pl.sl;                      // [nch][hi,lo] slot blocks
  float* part = reinterpret_cast<float*>(smb + pl.part);  // [T][65]   pool partials, then
  float* semc = part;                                     // [T][68]   the sem chunk
  unsigned char* xw = smb + pl.semc;                      // x block (hi, lo), then w block (hi, lo)

  __shared__ unsigned long long s_ticket;
  __shared__ long long s_pos;
  __shared__ int s_ok;
  __shared__ int s_bad;  // a staging wait ran out: skip global writes
  __shared__ float s_gpn[kTile + 1];  // gamma_far^n, n = 0 .. kTile
  __shared__ float s_gseg[kSeg];    // ema_gamma^(length) of the epilogue's token segments

  if (tid == 0) {
    for (int i = 0; i < 8; ++i) mbar_init(bars + i, 1);
    mbar_fence_init();
    s_bad = 0;
  }
  pdl_trigger();
  pdl_wait();

  // ---- ticket: the tile this cluster serves ----------------------------
  if (rank == 0 && tid == 0) s_ticket = atomicAdd(reinterpret_cast<unsigned long long*>(p.ws), 1ull);
  if (tid == 0) {
    const uint4 h0v = __ldcg(reinterpret_cast<const uint4*>(p.state));
    const uint4 h1v = __ldcg(reinterpret_cast<const uint4*>(p.state + 16));
    StateHeader hd;
    reinterpret_cast<uint4*>(&hd)[0] = h0v;
    reinterpret_cast<uint4*>(&hd)[1] = h1v;
    s_ok = (hd.magic == kMagic) & (hd.cfg_hash == p.cfg_hash) & (hd.batch == p.B) &
           (hd.n_layers == p.L);
  }
  cluster.sync();
  const long long ticket = static_cast<long long>(*cluster.map_shared_rank(&s_ticket, 0));
  if (!s_ok) {  // uniform over the whole grid: every CTA reads the same header
    if (tid == 0 && rank == 0 && ticket == 0) latch_error(p.err, SFA_ERR_STATE_MISMATCH);
    cluster.sync();  // rank 0's s_ticket must outlive the peers' reads
    return;
  }
  // Tensor memory for the pool accumulators (at most two CTAs per SM, so the
  // allocation never waits).
  if (warp == 0) tmem_alloc(tmem_slot, kTmemCols);

  const long long tile = ticket / p.n_streams;
  const int stream = static_cast<int>(ticket % p.n_streams);  // call-relative (layer, seq)
  const int l = p.l0 + stream / p.B;                          // layer of the state
  const bool last = (tile == p.tiles_per_stream - 1);
  const bool publish = (ticket != p.withhold_tile);
  const long long gstart = (tile / kGroup) * kGroup;         // first tile of this group
  const bool group_end = (tile % kGroup == kGroup - 1) && !last;

  unsigned char* blk = p.state + kHeaderBytes +
                      (static_cast<long long>(p.l0) * p.B + stream) * p.so.stride;
  if (tid == 0) s_pos = __ldcg(reinterpret_cast<const long long*>(blk + p.so.pos));
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
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

  // Slot of absolute position j >= 0 in the k-slot window.
  auto wslot = [&](long long j) -> long long { return j % K; };
  // Key row of absolute position j >= 0 for KV head g: from the input if it
  // belongs to this call, else from window slot j mod k (the state holds
  // positions pos0-k .. pos0-1).
  auto key_row = [&](long long j, int g) -> const Tin* {
    return (j >= pos0) ? kin + ((j - pos0) * nkv + g) * D : win_k + (wslot(j) * nkv + g) * D;
  };
  auto val_row = [&](long long j, int g) -> const Tin* {
    return (j >= pos0) ? vin + ((j - pos0) * nkv + g) * D : win_v + (wslot(j) * nkv + g) * D;
  };
  // Byte offset of element (c, d) in a packed [kSpan x D] key/value block:
  // 8 x 16-byte core matrices, the next span-row group 128 bytes on, the next
  // 8 dims kSpanR8 * 128 bytes on.  The same block is the K-major B of q·K^T
  // and the MN-major B of P·V.
  auto kv_off = [](int c, int d) -> int {
    return ((d >> 3) * kSpanR8 + (c >> 3)) * 128 + (c & 7) * 16 + (d & 7) * 2;
  };
  const int kvblk = kSpan * D * 2;
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
    unsigned bytes = tc ? 0u : 2u * row_bytes * valid;
    if (bi == 0) {
      if (!tc) bytes += static_cast<unsigned>(Tt * HS * ESZ);
      if (gstart == 0) bytes += static_cast<unsigned>(HS * 4);
      if (tile == 0)
        for (int r = 0; r < kHalo; ++r)
          if (t0 - kHalo + r >= 0) bytes += static_cast<unsigned>(HS * 4);
    }
    fence_proxy_async_smem();
    if (lane == 0) mbar_arrive_expect_tx(bar_kv, bytes);
    __syncwarp();
    for (int r = static_cast<int>(first_valid) + lane; r < (tc ? 0 : rows); r += 32) {
      const long long j = bs + r;
      const Tin* ks = (j >= pos0) ? kin + ((j - pos0) * nkv + g_lo) * D : win_k + (wslot(j) * nkv + g_lo) * D;
      const Tin* vs = (j >= pos0) ? vin + ((j - pos0) * nkv + g_lo) * D : win_v + (wslot(j) * nkv + g_lo) * D;
      bulk_g2s(kb + r * rowB, ks, row_bytes, bar_kv);
      bulk_g2s(vb + r * rowB, vs, row_bytes, bar_kv);
    }
    if (bi == 0) {
      for (int r = lane; r < (tc ? 0 : Tt); r += 32)
        bulk_g2s(qst + r * HS, qin + ((t0 - pos0 + r) * p.nq + h0) * D,
                 static_cast<unsigned>(HS * ESZ), bar_kv);
      // carries from the state, read before this tile publishes anything
      // (the stream's last tile overwrites them once all tiles have)
      if (gstart == 0 && lane == 0) bulk_g2s(fcar, field + rank * HS, static_cast<unsigned>(HS * 4), bar_kv);
      if (tile == 0 && lane < kHalo && t0 - kHalo + lane >= 0)
        bulk_g2s(halo + lane * HS, ring + static_cast<size_t>((t0 - kHalo + lane) % kRing) * p.H + rank * HS,
                 static_cast<unsigned>(HS * 4), bar_kv);
    }
  };
  issue_block(0);
  if (tile == 0)  // ring rows before position 0 are zero
    for (int idx = tid; idx < kHalo * HS; idx += NT)
      if (t0 - kHalo + idx / HS < 0) halo[idx] = 0.f;
  // Query block of head hh for the tensor-core near field: loads (rows past
  // the tile are zero) and packed stores [64 x D], split so the loads of the
  // next head overlap the current head's MMAs.
  constexpr int kQChunks = (kTile * (D / 8) + NT - 1) / NT;  // 16-byte chunks per thread
  auto q_load = [&](int hh, uint4 (&val)[kQChunks]) {
#pragma unroll
    for (int u = 0; u < kQChunks; ++u) {
      const int idx = u * NT + tid;
      const int d8 = idx / kTile, r = idx % kTile;
      val[u] = make_uint4(0u, 0u, 0u, 0u);
      if (idx < kTile * (D / 8) && r < Tt)
        val[u] = *reinterpret_cast<const uint4*>(qin + ((t0 - pos0 + r) * p.nq + h0 + hh) * D + d8 * 8);
    }
  };
  auto q_store = [&](const uint4 (&val)[kQChunks]) {
#pragma unroll
    for (int u = 0; u < kQChunks; ++u) {
      const int idx = u * NT + tid;
      if (idx < kTile * (D / 8)) *reinterpret_cast<uint4*>(qa + blk_off(idx % kTile, (idx / kTile) * 8)) = val[u];
    }
  };
  if constexpr (ESZ == 2) {
    if (tc) {
      // Head 0's query block and the key and value rows of the span
      // (positions t0-16 .. t0+63) for every KV head of the CTA, packed for
      // the MMAs; rows before position 0 or past the tile are zero.  One
      // pass of 16-byte loads, eight in flight per thread.
      constexpr int D8 = D / 8;
      const int per = kSpan * D8;
      const int nq_chunks = kTile * D8;
      const int total = nq_chunks + 2 * NG * per;
      for (int b0 = 0; b0 < total; b0 += 8 * NT) {
        uint4 val[8];
        int dst[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int idx = b0 + u * NT + tid;
          val[u] = make_uint4(0u, 0u, 0u, 0u);
          dst[u] = -1;
          if (idx < nq_chunks) {
            const int d8 = idx / kTile, r = idx % kTile;
            dst[u] = pl.qa + blk_off(r, d8 * 8);  // offsets from the shared-memory base
            if (r < Tt)
              val[u] = *reinterpret_cast<const uint4*>(qin + ((t0 - pos0 + r) * p.nq + h0) * D + d8 * 8);
          } else if (idx < total) {
            const int kvi = idx - nq_chunks;
            const int which = kvi / (NG * per), rem = kvi % (NG * per);
            const int gg = rem / per, r2 = rem % per;
            const int d8 = r2 / kSpan, c = r2 % kSpan;
            const long long j = kv_start + c;
            dst[u] = pl.kvp + (which * p.NGm + gg) * kvblk + kv_off(c, d8 * 8);
            if (j >= 0 && c < kv_rows) {
              const Tin* row = which ? val_row(j, g_lo + gg) : key_row(j, g_lo + gg);
              val[u] = *reinterpret_cast<const uint4*>(row + d8 * 8);
            }
          }
        }
#pragma unroll
        for (int u = 0; u < 8; ++u)
          if (dst[u] >= 0) *reinterpret_cast<uint4*>(smb + dst[u]) = val[u];
      }
      for (int i = tid; i < 2 * kTile * kSpan * 2 / 16; i += NT)  // P blocks start at zero
        reinterpret_cast<uint4*>(pa)[i] = make_uint4(0u, 0u, 0u, 0u);
    }
  }
  if (!tc)  // running state of the near field (overlaps the copies in flight)
    for (int i = tid; i < kTile * HPC; i += NT) {
      mrun[i] = -INFINITY;
      lrun[i] = 0.f;
    }
  for (int i = tid; i < kTile * XS; i += NT) xs[i] = 0.f;
  if (!mbar_wait_bounded(bar_kv, 0, kMbarPollLimit, p.err)) s_bad = 1;
  __syncthreads();  // the packed blocks and zeroed rows written above are read by other threads
  // Keys that leave the window at the tile's tokens are rows 0 .. Tt-1 of the
  // staged span when the first block covers them; otherwise read them from
  // global memory.
  bool ev_staged = tc || p.KB >= Tt;
  // Folds the keys that leave the window at tokens r of [r_lo, r_hi) with
  // r >= r_from into s (EWMA), calling visit(r, s) after every token; staged
  // rows or global memory.
  auto scan_evicted = [&](int gg, int i, int r_lo, int r_hi, int r_from, float s,
                          auto&& visit) -> float {
    if (ev_staged && tc) {  // packed key block: span row r is position t0 - k + r
      const unsigned char* kg = kvp + gg * kvblk;
      for (int r = r_lo; r < r_hi; ++r) {
        if (r >= r_from) s = ewma(gf, s, to_f32<Tin>(*reinterpret_cast<const Tin*>(kg + kv_off(r, i))));
        visit(r, s);
      }
    } else if (ev_staged) {
      const Tin* col = reinterpret_cast<const Tin*>(kb) + gg * D + i;
      const int pitch = rowB / ESZ;
      for (int r = r_lo; r < r_hi; ++r) {
        if (r >= r_from) s = ewma(gf, s, to_f32<Tin>(col[r * pitch]));
        visit(r, s);
      }
    } else {
      for (int r0 = r_lo; r0 < r_hi; r0 += kEvChunk) {
        float ev[kEvChunk];
#pragma unroll
        for (int u = 0; u < kEvChunk; ++u)
          ev[u] = (r0 + u < r_hi && r0 + u >= r_from) ? to_f32<Tin>(key_row(t0 + r0 + u - K, g_lo + gg)[i]) : 0.f;
#pragma unroll
        for (int u = 0; u < kEvChunk; ++u) {
          const int r = r0 + u;
          if (r < r_hi) {
            if (r >= r_from) s = ewma(gf, s, ev[u]);
            visit(r, s);
          }
        }
      }
    }
    return s;
  };

  // ---- (A) far field: this tile's aggregate of the keys leaving the window.
  // The tile's tokens split into nseg (1, 2 or 4) segments per (KV head, dim)
  // as the threads allow; each segment is folded from zero, then the
  // segments are combined in order: fold(c, seg) = gamma^(evictions) c + agg.
  const int r_ev = static_cast<int>(max(0LL, min(static_cast<long long>(Tt), K - t0)));  // first token that evicts
  const int ne = NG * D;
  int nseg = 1;
  while (nseg < 4 && ne * nseg * 2 <= NT) nseg *= 2;
  const int seg_len = kTile / nseg;
  auto seg_ev = [&](int sg) -> int {  // evicting tokens of segment sg
    const int a = max(sg * seg_len, r_ev), b = min(Tt, (sg + 1) * seg_len);
    return b > a ? b - a : 0;
  };
  if (tid <= kTile) s_gpn[tid] = powf(gf, static_cast<float>(tid));
  if (tid < ne * nseg) {
    const int elem = tid % ne, sg = tid / ne;
    segA[sg * ne + elem] = scan_evicted(elem / D, elem % D, sg * seg_len, min(Tt, (sg + 1) * seg_len),
                                        r_ev, 0.f, [](int, float) {});
  }
  __syncthreads();
  for (int idx = tid; idx < ne; idx += NT) {
    const int g = g_lo + idx / D, i = idx % D;
    float a = 0.f;
    for (int sg = 0; sg < nseg; ++sg) a = fmaf(s_gpn[seg_ev(sg)], a, segA[sg * ne + idx]);
    sagg[idx] = a;
    if (g >= own_lo && publish) agg_s[(ticket * nkv + g) * D + i] = a;
  }
  __syncthreads();
  if (tid == 0 && publish) {
    __threadfence();
    for (int g = own_lo; g <= g_hi; ++g) st_release_u32(&fs_agg[ticket * nkv + g], 1u);
  }

  // ---- (B) near field [P1 §2.1 eq. O_near] ---------------------------------
  bool near_done = false;
  if constexpr (ESZ == 2) {
    if (tc) {
      // On the tensor cores, one query head at a time:
      //   S[64 x kSpan] = Q_h . K_g^T (tensor memory, columns 0..kSpan-1);
      //   softmax over the band of each row (token r sees span rows r+1 ..
      //   r+k, positions t0+r-k+1 .. t0+r, none before position 0);
      //   P split into bf16 hi + lo (about 16 significant bits);
      //   O[64 x D] = P_hi . V_g + P_lo . V_g (columns kTmemO..), into the x tile.
      // Accumulator row r sits in lane (r % 16) + 32 (r / 16); warp w (w < 4)
      // loads span columns 32 (w / 2) .. + 63, which hold the bands of its 16 rows.
      const uint32_t idesc_qk = umma_idesc_bf16(kTile, kSpan, false);
      const uint32_t idesc_pv = umma_idesc_bf16(kTile, D, true);
      const int sp = warp & 3, pbase = 32 * (sp >> 1);
      const int cmin = kv_start < 0 ? static_cast<int>(-kv_start) : 0;  // first row at position >= 0
      unsigned char* pa_hi = pa;
      unsigned char* pa_lo = pa + kTile * kSpan * 2;
      unsigned nf_par = 0;
      for (int hh = 0; hh < HPC; ++hh) {
        const int gg = (h0 + hh) / G - g_lo;
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
          tc_fence_after();
          const unsigned char* kg = kvp + gg * kvblk;
#pragma unroll
          for (int s2 = 0; s2 < D / 16; ++s2)
            umma_bf16(tmem, umma_desc(qa + s2 * 2048, 1024, 128),
                      umma_desc(kg + s2 * 2 * kSpanR8 * 128, kSpanR8 * 128, 128), idesc_qk, s2 > 0);
          umma_commit(bar_nf);
        }
        uint4 qn[kQChunks];  // the next head's queries, in flight during the MMAs
        if (hh + 1 < HPC) q_load(hh + 1, qn);
        if (!mbar_wait_bounded(bar_nf, nf_par, kMbarPollLimit, p.err)) s_bad = 1;
        nf_par ^= 1u;
        tc_fence_after();
        if (hh + 1 < HPC) q_store(qn);  // the score MMAs have read the query block
        if (warp < 4) {
          float v[64];
          tmem_ld32(tmem + (static_cast<uint32_t>(32 * sp) << 16) + pbase, *reinterpret_cast<float(*)[32]>(v));
          tmem_ld32(tmem + (static_cast<uint32_t>(32 * sp) << 16) + pbase + 32,
                    *reinterpret_cast<float(*)[32]>(v + 32));
          // The bands of rows 16 sp .. 16 sp + 15 lie in span columns
          // 16 sp .. 16 sp + 31: loaded columns J0 .. J0 + 31 with
          // J0 = 16 (sp & 1); only those are scored and written (the other
          // P columns stay zero).
          auto band = [&](auto j0_c) {
            constexpr int J0 = decltype(j0_c)::value;
            const int r = 16 * sp + lane;
            float mx = -INFINITY;
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const int c = pbase + J0 + j;
              const bool in = c >= r + 1 && c <= r + K && c >= cmin;
              v[J0 + j] = in ? v[J0 + j] * p.score_scale : -INFINITY;
              mx = fmaxf(mx, v[J0 + j]);
            }
            float sum = 0.f;
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              v[J0 + j] = __expf(v[J0 + j] - mx);  // 0 outside the band
              sum += v[J0 + j];
            }
            const float inv = 1.f / sum;
#pragma unroll
            for (int g8 = 0; g8 < 4; ++g8) {
              uint32_t hw[4], lw[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                __nv_bfloat16 h0b, l0b, h1b, l1b;
                split_bf16(v[J0 + 8 * g8 + 2 * e] * inv, h0b, l0b);
                split_bf16(v[J0 + 8 * g8 + 2 * e + 1] * inv, h1b, l1b);
                hw[e] = static_cast<uint32_t>(__bfloat16_as_ushort(h0b)) |
                        (static_cast<uint32_t>(__bfloat16_as_ushort(h1b)) << 16);
                lw[e] = static_cast<uint32_t>(__bfloat16_as_ushort(l0b)) |
                        (static_cast<uint32_t>(__bfloat16_as_ushort(l1b)) << 16);
              }
              const int off = blk_off(r, pbase + J0 + 8 * g8);
              *reinterpret_cast<uint4*>(pa_hi + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
              *reinterpret_cast<uint4*>(pa_lo + off) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
            }
          };
          if (lane < 16) {
            if (sp & 1) band(std::integral_constant<int, 16>{});
            else band(std::integral_constant<int, 0>{});
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {
          tc_fence_after();
          const unsigned char* vg = kvp + (p.NGm + gg) * kvblk;
#pragma unroll
          for (int s2 = 0; s2 < kSpan / 16; ++s2) {
            const uint64_t bv = umma_desc(vg + s2 * 256, 128, kSpanR8 * 128);
            umma_bf16(tmem + kTmemO, umma_desc(pa_hi + s2 * 2048, 1024, 128), bv, idesc_pv, s2 > 0);
            umma_bf16(tmem + kTmemO, umma_desc(pa_lo + s2 * 2048, 1024, 128), bv, idesc_pv, true);
          }
          umma_commit(bar_nf);
        }
        if (!mbar_wait_bounded(bar_nf, nf_par, kMbarPollLimit, p.err)) s_bad = 1;
        nf_par ^= 1u;
        tc_fence_after();
        {  // O rows into the x tile: warps w and w + 4 take halves of the head
          const int colh = (warp >> 2) * (D / 2);
          const int r = 16 * sp + lane;
#pragma unroll
          for (int c0 = 0; c0 < D / 2; c0 += 32) {
            float v[32];
            tmem_ld32(tmem + (static_cast<uint32_t>(32 * sp) << 16) + kTmemO + colh + c0, v);
            if (lane < 16 && r < Tt) {
              float* dst = xs + r * XS + hh * D + colh + c0;
#pragma unroll
              for (int j = 0; j < 32; j += 4)
                *reinterpret_cast<float4*>(dst + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
            }
          }
        }
        tc_fence_before();
        __syncthreads();
      }
      near_done = true;
    }
  }
  if (!near_done) {  // on the CUDA cores, block by block
    for (int bi = 0; bi < n_blocks; ++bi) {
      if (bi > 0 && !mbar_wait_bounded(bar_kv, bi & 1, kMbarPollLimit, p.err)) s_bad = 1;
      const long long bs = kv_start + static_cast<long long>(bi) * p.KB;
      const long long be = bs + min(p.KB, kv_rows - bi * p.KB);  // exclusive
      if (K <= 16)
        near_block<Tin, D, 16>(qst, kb, vb, xs, mrun, lrun, rowB, HS, XS, HPC, G, g_lo, K, t0, Tt,
                               bs, be, p.score_scale, h0, warp, lane);
      else
        near_block<Tin, D, 32>(qst, kb, vb, xs, mrun, lrun, rowB, HS, XS, HPC, G, g_lo, K, t0, Tt,
                               bs, be, p.score_scale, h0, warp, lane);
      __syncthreads();  // the block buffers are free again
      if (bi + 1 < n_blocks) issue_block(bi + 1);
    }
    if (n_blocks > 1) ev_staged = false;  // the staged rows were replaced by later blocks
    // normalise: O = acc / den
    for (int i = tid; i < Tt * HPC; i += NT) lrun[i] = 1.f / lrun[i];
    __syncthreads();
    for (int r = warp; r < Tt; r += NW)
      for (int c = lane; c < HS; c += 32) xs[r * XS + c] *= lrun[r * HPC + c / D];
  }

  // ---- (C) far field carry-in (deterministic look-back), then the scan --
  // carry = INCL(end of previous group) or the state, folded with the
  // aggregates of the group's earlier tiles in order.  Warp 0 polls all the
  // flags at once (lane per flag); then every carry element loads all its
  // terms at once and folds them in order.
  const int n_prev = static_cast<int>(tile - gstart);  // earlier tiles of the group (< kGroup)
  {
    if (warp == 0) {
      const int n_flags = (n_prev + (gstart > 0 ? 1 : 0)) * NG;
      for (int f = lane; f < n_flags; f += 32) {
        const int gg = f % NG, jj = f / NG;
        const unsigned* fl = (jj < n_prev) ? &fs_agg[ticket_of(gstart + jj) * nkv + g_lo + gg]
                                           : &fs_incl[ticket_of(gstart - 1) * nkv + g_lo + gg];
        wait_flag(fl, p.spin_limit, p.err);
      }
    }
    __syncthreads();
    for (int idx = tid; idx < NG * D; idx += NT) {
      const int g = g_lo + idx / D, i = idx % D;
      float terms[kGroup];
#pragma unroll
      for (int jj = 0; jj < kGroup - 1; ++jj)
        terms[jj] = (jj < n_prev) ? __ldcg(agg_s + (ticket_of(gstart + jj) * nkv + g) * D + i) : 0.f;
      float acc = (gstart == 0) ? far[g * D + i] : __ldcg(incl_s + (ticket_of(gstart - 1) * nkv + g) * D + i);
#pragma unroll
      for (int jj = 0; jj < kGroup - 1; ++jj)
        if (jj < n_prev)
          acc = fmaf(s_gpn[evictions(pos0 + (gstart + jj) * kTile, kTile)], acc, terms[jj]);
      sst[idx] = acc;
    }
    __syncthreads();
    if (group_end && publish) {
      const float mul = s_gpn[evictions(t0, Tt)];
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
  // scan: S_t per token, x = O_near + alpha_far * S_t  [P1 §2.1 eq. O];
  // segment sg starts from the carry folded with the earlier segments'
  // aggregates.  The last segment leaves S at the tile end in its own
  // segA entry, which no other thread reads.
  if (tid < ne * nseg) {
    const int elem = tid % ne, sg = tid / ne;
    const int gg = elem / D, i = elem % D, g = g_lo + gg;
    const int hh_lo = max(0, g * G - h0), hh_hi = min(HPC, (g + 1) * G - h0);
    float c = sst[elem];
    for (int s2 = 0; s2 < sg; ++s2) c = fmaf(s_gpn[seg_ev(s2)], c, segA[s2 * ne + elem]);
    c = scan_evicted(gg, i, sg * seg_len, min(Tt, (sg + 1) * seg_len), r_ev, c,
                     [&](int r, float sv) {
                       for (int hh = hh_lo; hh < hh_hi; ++hh) {
                         float* xp = xs + r * XS + hh * D + i;
                         *xp = fmaf(p.alpha_far, sv, *xp);
                       }
                     });
    if (sg == nseg - 1) segA[sg * ne + elem] = c;
  }
  __syncthreads();
  // Slot blocks (bf16 hi/lo, laid out for both pool MMAs); the staging
  // buffers are free now.
  const unsigned char* img = p.slot_img +
      (static_cast<size_t>(l) * (p.H / kBlk) + static_cast<size_t>(rank) * nch) * 2 * kBlkBytes;
  if (tid == 0) {
    fence_proxy_async_smem();
    mbar_arrive_expect_tx(bar_sl, static_cast<unsigned>(nch * 2 * kBlkBytes));
    for (int c = 0; c < nch; ++c)
      bulk_g2s(simg + c * 2 * kBlkBytes, img + static_cast<size_t>(c) * 2 * kBlkBytes,
               2u * kBlkBytes, bar_sl);
  }

  // ---- (D) EMA field aggregate; tail rows for the successor -------------
  // (Tiles of the first group staged the state field, and tile 0 the state
  // ring rows, with the first key block.)
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

  // ---- (E) pool scores on the tensor cores [P3 §2.1 channel 3] -----------
  // scores[T x 64] (tensor memory, columns 0..63) = sum over 64-column chunks
  // of x_chunk . slot_chunk^T, each as hi*hi + hi*lo + lo*hi.
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
      for (int s = 0; s < kBlk / 16; ++s) {
        const uint64_t ah = umma_desc(xhi + s * 2048, 1024, 128), al = umma_desc(xlo + s * 2048, 1024, 128);
        const uint64_t bh = umma_desc(shi + s * 2048, 1024, 128), bl = umma_desc(slo + s * 2048, 1024, 128);
        umma_bf16(tmem, ah, bh, idesc_s, c > 0 || s > 0);
        umma_bf16(tmem, ah, bl, idesc_s, true);
        umma_bf16(tmem, al, bh, idesc_s, true);
      }
      umma_commit(bar_ms);
    }
  }
  if (tid == 0) umma_commit(bar_sd);
  // |x|^2 per token (CUDA cores) while the tensor cores finish
  for (int r = warp; r < kTile; r += NW) {
    float ss = 0.f;
    for (int e = lane; e < HS; e += 32) ss = fmaf(xs[r * XS + e], xs[r * XS + e], ss);
    ss = warp_sum(ss);
    if (lane == 0) part[r * kPartStride + kSlots] = ss;
  }
  if (!mbar_wait_bounded(bar_sd, 0, kMbarPollLimit, p.err)) s_bad = 1;
  tc_fence_after();
  {  // accumulator row r (token) sits in lane (r%16) + 32*(r/16) for M = 64
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

  // ---- (F) EMA field carry-in (deterministic look-back); tail rows ------
  {
    if (warp == 0) {
      const int n_flags = n_prev + (gstart > 0 ? 1 : 0);
      for (int f = lane; f < n_flags; f += 32) {
        const unsigned* fl = (f < n_prev) ? &ff_agg[ticket_of(gstart + f) * p.CS + rank]
                                          : &ff_incl[ticket_of(gstart - 1) * p.CS + rank];
        wait_flag(fl, p.spin_limit, p.err);
      }
      // the predecessor's tail rows come with its aggregate (or, across a
      // group boundary, with the inclusive value published after it)
    }
    __syncthreads();
    const float mul_full = powf(ge, static_cast<float>(kTile));
    for (int e = tid; e < HS; e += NT) {
      float terms[kGroup];
#pragma unroll
      for (int jj = 0; jj < kGroup - 1; ++jj)
        terms[jj] = (jj < n_prev) ? __ldcg(agg_f + ticket_of(gstart + jj) * p.H + rank * HS + e) : 0.f;
      float acc = (gstart == 0) ? fcar[e] : __ldcg(incl_f + ticket_of(gstart - 1) * p.H + rank * HS + e);
#pragma unroll
      for (int jj = 0; jj < kGroup - 1; ++jj)
        if (jj < n_prev) acc = fmaf(mul_full, acc, terms[jj]);
      fcar[e] = acc;
    }
    if (tile > 0)  // x rows of the 15 tokens before the tile, from the predecessor
      for (int idx = tid; idx < kHalo * HS; idx += NT) {
        const int r = idx / HS, e = idx % HS;
        halo[idx] = __ldcg(halo_ws + (ticket_of(tile - 1) * kHalo + r) * p.H + rank * HS + e);
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
      // every rank's partials in flight at once, added in rank order
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
      __nv_bfloat16 h0, l0, h1, l1;
      split_bf16(e0 * inv, h0, l0);
      split_bf16(e1 * inv, h1, l1);
      const int o0 = blk_off(r, lane), o1 = blk_off(r, lane + 32);
      for (int q = 0; q < p.CS; ++q) {
        unsigned char* wq = cluster.map_shared_rank(xw, q);  // the x blocks are dead everywhere
        *reinterpret_cast<__nv_bfloat16*>(wq + o0) = h0;
        *reinterpret_cast<__nv_bfloat16*>(wq + kBlkBytes + o0) = l0;
        *reinterpret_cast<__nv_bfloat16*>(wq + o1) = h1;
        *reinterpret_cast<__nv_bfloat16*>(wq + kBlkBytes + o1) = l1;
      }
    }
    // rows of tokens past the tile end feed MMA rows that are never read
    fence_proxy_async_cluster();
  }
  cluster.sync();

  // ---- (H) semantic mix on the tensor cores, then per column chunk: ring,
  // field, fusion, clip, output [P3 §2.1 channels 1–3, §2.2].
  // sem chunk c [T x 64] = w[T x 64] . slot_chunk_c, accumulators alternate
  // between tensor-memory columns 64..127 and 128..191.
  unsigned char* whi = xw;  // written by the cluster in (G)
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
    for (int s = 0; s < kSlots / 16; ++s) {
      const uint64_t ah = umma_desc(whi + s * 2048, 1024, 128), al = umma_desc(wlo + s * 2048, 1024, 128);
      const uint64_t bh = umma_desc(shi + s * 256, 128, 1024), bl = umma_desc(slo + s * 256, 128, 1024);
      umma_bf16(dst, ah, bh, idesc_c, s > 0);
      umma_bf16(dst, ah, bl, idesc_c, true);
      umma_bf16(dst, al, bh, idesc_c, true);
    }
    umma_commit(bar_mc + (c & 1));
  };
  if (tid == 0) {
    issue_sem(0);
    if (nch > 1) issue_sem(1);
  }
  const float a_l = p.alpha_layer[l];
  const bool write_ok = !s_bad;
  if (tid < kSeg) {
    const int len = max(0, min(Tt, (tid + 1) * (kTile / kSeg)) - tid * (kTile / kSeg));
    s_gseg[tid] = powf(ge, static_cast<float>(len));
  }  // read after the first barrier of the chunk loop below
  float* out = p.out + (in_row0 + (t0 - pos0)) * p.H + rank * HS;
  for (int c = 0; c < nch; ++c) {
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
    // field: per-segment aggregates, then carries folded in segment order
    const int cc = tid % kCW, sg = tid / kCW;  // column, token segment
    const int e = c * kCW + cc;
    const int r_lo = sg * (kTile / kSeg), r_hi = min(Tt, r_lo + kTile / kSeg);
    {
      float a = 0.f;
      for (int r = r_lo; r < r_hi; ++r) a = ewma(ge, a, xs[r * XS + e]);
      segc[sg * kCW + cc] = a;
    }
    __syncthreads();
    float f = fcar[e];
    for (int s2 = 0; s2 < sg; ++s2) f = fmaf(s_gseg[s2], f, segc[s2 * kCW + cc]);
    // ring: sum of the 16 positions ending at r, from the x tile and the halo
    auto xat = [&](int r) -> float { return r >= 0 ? xs[r * XS + e] : halo[(r + kHalo) * HS + e]; };
    float rs = 0.f;
    if (r_lo < r_hi)
      for (int r = r_lo - kHalo; r <= r_lo; ++r) rs += xat(r);
    for (int r = r_lo; r < r_hi; ++r) {
      if (r > r_lo) rs += xat(r) - xat(r - kRing);
      const float x = xs[r * XS + e];
      f = ewma(ge, f, x);
      float u = rs * (1.0f / kRing) + 0.5f * f + 0.5f * semc[r * kSemStride + cc];
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
      if (g >= own_lo) far[g * D + i] = segA[(nseg - 1) * ne + idx];  // S at the tile end
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
        const long long dst = (wslot(j) * nkv + g) * D + i;
        win_k[dst] = kin[src];
        win_v[dst] = vin[src];
      }
    }
    if (rank == 0 && tid == 0) *reinterpret_cast<long long*>(blk + p.so.pos) = pos0 + p.n;
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

}  // namespace

// Shared-memory plan: persistent regions, then a union of the staging
// buffers (near-field phase) and the pool buffers (pool phase).  The key
// block is as tall as fits, up to the whole span t0-k .. t0+T-1.  The plan
// never drops below a third of the SM's shared memory, so at most two CTAs
// share an SM and their tensor-memory allocations (256 columns each) always
// fit at once.
bool plan_prefill(int HPC, int D, int esz, int NGm, int K, size_t budget, bool tc,
                  PrefillPlan* out) {
  const int HS = HPC * D, XS = HS + 4;
  if (HS % kBlk != 0) return false;
  if (tc && (esz != 2 || K > kSpan - kTile)) return false;
  auto a16 = [](long long x) { return static_cast<int>((x + 15) & ~15LL); };
  PrefillPlan p;
  std::memset(&p, 0, sizeof(p));
  p.tc = tc ? 1 : 0;
  int off = 0;
  p.bars = off;                 off += 128;  // mbarriers and the tensor-memory address
  p.xs = off;                   off += a16(4LL * kTile * XS);
  p.halo = off;                 off += a16(4LL * kHalo * HS);
  p.fcar = off;                 off += a16(4LL * HS);
  p.sst = off;                  off += a16(4LL * NGm * D);
  p.sagg = off;                 off += a16(4LL * NGm * D);
  p.sega = off;                 off += a16(4LL * NT);   // far-field scan segments
  // epilogue carries, then (CUDA-core near field) running max / denominator
  p.ml = off;                   off += a16(4LL * (kSeg * kCW + (tc ? 0 : 2 * kTile * HPC)));
  p.u0 = off;
  // pool phase: slot blocks, partials | sem chunk, x block | w block
  int q = off;
  p.sl = q;                     q += a16(static_cast<long long>(HS / kBlk) * 2 * kBlkBytes);
  p.part = q;                   q += a16(4LL * kTile * std::max(kPartStride, kSemStride));
  p.wts = q;
  p.semc = q;                   q += a16(2LL * kBlkBytes);
  const int pool_end = q;
  q = off;
  if (tc) {
    // near-field phase on the tensor cores: one query block, key and value
    // blocks of every KV head of the CTA, the P block (hi, lo)
    p.qa = q;                   q += a16(2LL * kTile * D);
    p.kvp = q;                  q += a16(2LL * 2 * NGm * kSpan * D);
    p.pa = q;                   q += a16(2LL * 2 * kTile * kSpan);
    p.KB = kSpan;
  } else {
    // near-field phase on the CUDA cores: staged queries and key/value rows
    p.qst = q;                  q += a16(static_cast<long long>(kTile) * HS * esz);
    const int row_b = NGm * D * esz + 16;
    const long long room = static_cast<long long>(budget) - q;
    int kb_rows = static_cast<int>(room / (2LL * row_b));
    kb_rows = std::min(kb_rows, kTile + K);
    if (kb_rows < 32) return false;
    p.KB = kb_rows;
    p.kb = q;                   q += a16(static_cast<long long>(row_b) * kb_rows);
    p.vb = q;                   q += a16(static_cast<long long>(row_b) * kb_rows);
  }
  p.total = std::max(q, pool_end);
  p.total = std::max<int>(p.total, static_cast<int>((budget + 1024) / 3) + 1);
  if (static_cast<size_t>(p.total) > budget) return false;
  *out = p;
  return true;
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
