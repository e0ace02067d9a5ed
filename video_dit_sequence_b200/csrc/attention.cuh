// attention.cuh -- full-sequence, non-causal bf16 attention per head on
// tcgen05 tensor cores (sm_100a).
//
// What it computes (fal.ai "Generate video with WAN 2.2 across four GPUs",
// section "Splitting one generation across four GPUs": after the exchange
// each rank attends over the full sequence for its heads):
//   O[i] = sum_{k<N} softmax_k(q_i . k_k * scale) v_k      for i < N,
//   O[i] = 0                                               for N <= i < Np.
// The softmax is evaluated online, one 128-key tile at a time (flash
// attention), which reaches the two-pass result up to rounding.
//
// One CTA owns two 128-row query tiles of one (batch, head).  Roles:
//   warps 0-3  softmax for query tile 0 (one thread per query row)
//   warps 4-7  softmax for query tile 1
//   warp  8    TMA producer: Q once, then K_j, V_j into a ring of smem slots
//   warp  9    TMEM allocator and the single MMA-issuing thread
// Tensor memory (512 columns x 128 lanes, fp32): S_t at columns 128t,
// O_t at columns 256 + D*t.  The softmax writes P_t (bf16, two per column)
// over the first 64 columns of S_t, and the P*V product reads it from there.
// Per key tile j the MMA thread issues, in this order,
//   O_0 += P_0 V_j,  S_0 = Q_0 K_{j+1}^T,  O_1 += P_1 V_j,  S_1 = Q_1 K_{j+1}^T
// so the tensor core works on one query tile while the other one's softmax
// runs.  tcgen05 operations from one thread execute in issue order, so an S
// write never overtakes the P read before it, and the commit that signals
// "S_{t,j+1} ready" also covers the O_t update before it: when a softmax
// thread sees S ready it may rescale O_t in place.
//
// Online softmax with a lazily updated row maximum: the running reference
// m (log2 units) moves only when a tile's maximum exceeds it by more than 8,
// so probabilities stay <= 2^8 and O is rescaled rarely.  The arithmetic of
// a row depends only on its own scores and the fixed key-tile order, never on
// P, the layout, or the CTA it runs in: outputs are bit-identical across
// degrees and between the fused and the three-call path.
//
// One body serves three kernels: bf16 (D = 64 or 128), E4M3 operands with
// per-block / per-channel scale factors (kF8), and one rank's step of the
// multi-GPU form (kPeer), which reads Q tiles from, and stores O rows into,
// the shards of the ranks that hold those tokens.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "sm100.cuh"

namespace sp {

struct AttnParams {
  int32_t N;            // true tokens (keys and queries)
  int32_t Np;           // rows that exist in the output buffer per (batch, head)
  int32_t H;            // global heads
  int32_t B;
  int32_t hsplit;       // heads per tensor-map "batch" slot (Hl or H)
  int32_t num_kv_tiles; // ceil(N / 128)
  float scale_log2e;    // scale * log2(e)
  __nv_bfloat16 *o;     // output base
  int64_t o_row;        // elements between consecutive tokens
  int64_t o_batch;      // elements between tensor-map batch slots
  // Rank-major sequence shards with B > 1 and P > 1 ([P][B][Nl][H][D]):
  // nl_split = Nl (else 0); token t lives in rank t / Nl at local row t % Nl.
  int32_t nl_split;
  int64_t o_rank;       // elements between rank slabs (B * Nl * H * D)
  const uint8_t *q, *k, *v;  // bases, for tiles that cross a shard boundary
  // E4M3 variant: scale factors, element value = byte value * factor.
  // dq, dk: [B][H][nblk], one per block of 128 tokens (= one query or key
  // tile); dv: [B][H][D], one per channel.  Null for bf16.
  const float *dq, *dk, *dv;
  int32_t nblk;
  float *lse;           // [B][H][Np] or null
  int32_t *status;      // device status word
  // Block-sparse variant: mask [B][H][ncube][nwords] bits over cubes of 64
  // tokens; bit c of word w in query cube qc's row selects key cube 32w + c.
  const uint32_t *mask;
  int32_t ncube, nwords;
  // Peer step with the K/V exchange overlapped (null: everything has
  // arrived before the launch).  counts[r] counts the finished pieces of
  // source rank r's K/V chunk (and, through stream order on rank r, covers
  // its Q shard); the chunk has arrived when counts[r] >= count_target.
  // Tokens of chunk r are r*count_nl .. r*count_nl + count_nl - 1.
  const unsigned long long *counts;
  unsigned long long count_target;
  int32_t count_nl;
  uint64_t count_wait_ns;
};

constexpr int32_t kStatusTimeout = 7;

// One rank's step of the multi-GPU form with the Q and O exchanges fused
// into the kernel: rank r's sequence shard of Q and its output shard O are
// [B][Nl][H][D] bf16 on GPU r, reached through peer addresses.  Query token
// t of the head group lives in rank t / nl at local row t % nl; this rank
// attends heads head0 .. head0 + Hl - 1 of the H global heads.
constexpr int kMaxPeers = 8;
struct PeerArgs {
  CUtensorMap q[kMaxPeers];            // 4-D maps (D, H, Nl, B) over each rank's Q shard
  const uint8_t *q_ptr[kMaxPeers];     // the same shards, for tiles that cross ranks
  __nv_bfloat16 *o_ptr[kMaxPeers];     // each rank's output shard
  int32_t nranks;                      // P
  int32_t nl;                          // tokens per rank
  int32_t heads;                       // H, global heads of a shard row
  int32_t head0;                       // first global head of this rank's group
};

// kF8: operands in E4M3 (one byte) instead of bf16 (two bytes).
template <int D, bool kF8 = false>
struct AttnCfg {
  static_assert(D == 64 || D == 128, "head dim");
  static_assert(!kF8 || D == 128, "the E4M3 variant has D = 128");
  static constexpr int kBM = 128;                   // query rows per tile
  static constexpr int kBN = 128;                   // keys per tile
  static constexpr int kElemBytes = kF8 ? 1 : 2;
  static constexpr int kRowBytes = D * kElemBytes;  // one token row of one head
  static constexpr int kHalves = kRowBytes / 128;   // 128-byte column blocks per row
  static constexpr int kBoxInner = 128 / kElemBytes;  // elements per 128-byte block row
  static constexpr int kBlockBytes = 128 * 128;     // 128 rows x 128 bytes (one swizzle block)
  static constexpr int kTileBytes = kHalves * kBlockBytes;
  static constexpr int kQkSteps = kRowBytes / 32;   // MMA K steps of 32 bytes over D
  static constexpr int kPvKeys = 32 / kElemBytes;   // keys per PV MMA (K = 16 or 32)
  static constexpr int kPvSteps = kBN / kPvKeys;
  static constexpr int kPCols = kBN * kElemBytes / 4;  // TMEM columns of one P row
  // Probabilities are 2^(s*scale*log2e - m + kShift) and the reference m
  // moves when a tile maximum exceeds it by more than kThresh, so they stay
  // below 2^(kThresh + kShift): 2^8 for both.  E4M3 keeps 3 mantissa bits
  // above 2^-6 only; the shift of 6 lifts the typical weights of a long
  // sequence (about 2^-6 of the row maximum) out of its subnormal range.
  static constexpr float kShift = kF8 ? 6.0f : 0.0f;
  static constexpr float kThresh = kF8 ? 2.0f : 8.0f;
  static constexpr int kStages = 4;
  static constexpr int kOffQ = 0;
  static constexpr int kOffKV = 2 * kTileBytes;
  static constexpr int kOffBar = kOffKV + kStages * kTileBytes;
  static constexpr int kNumBar = 1 + 2 * kStages + 9;  // ..., bar_o[2], bar_drain
  static constexpr int kOffMisc = kOffBar + kNumBar * 8;
  // Misc: TMEM base, abort flag, per ring slot the index of the last load
  // issued into it (-1: none), then the block-sparse plan's two list lengths.
  static constexpr int kOffCount = kOffMisc + 16 + 4 * kStages;
  static constexpr int kOffPlan = kOffCount + 16;
  static constexpr int kSmemBytes = kOffPlan + 1024;  // + alignment slack
  // Block-sparse plan: per query tile, the 64-token key cubes it visits as
  // 16-bit indices (and a closing ncube when their number is odd).
  static constexpr int kMaxPlanCubes = 8192;
  static constexpr int kPlanStride = kMaxPlanCubes + 2;
  static constexpr int kSmemBytesSparse = kOffPlan + 2 * 2 * kPlanStride + 1024;
  static_assert(kSmemBytesSparse <= 227 * 1024, "shared memory per CTA");
  static constexpr int kThreads = 320;
  static constexpr uint32_t kColS1 = 128;
  static constexpr uint32_t kColO0 = 256;
  static constexpr uint32_t kColO1 = 256 + D;
  static constexpr uint32_t kTmemCols = 512;
};

constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s per wait


// Rows r0 .. r0 + nrows - 1 of a K/V or Q tile in shared memory at dst take
// tokens t0 .. t0 + nrows - 1 of the rank-major layout [P][B][nl][H][row]
// (zeros past N), in the 128-byte-swizzled layout the TMA writes: 16-byte
// chunk c of row r at chunk c ^ (r mod 8) of its column block.  The whole
// warp copies with 16-byte loads, then fences the generic-proxy writes for
// the async proxy.  Out of line: the path is rare (a tile or cube that
// crosses a shard boundary) and each inlined copy would grow the hot code.
// kCoherent: plain loads (data another GPU may still be writing), else
// non-coherent ones.
template <int kRowBytes, bool kCoherent>
__device__ __noinline__ void copy_rows(const uint8_t *base, uint32_t dst, int t0, int r0, int nrows,
                                       int N, int nl, int B, int b, int H, int head, int lane) {
  constexpr int kChunks = kRowBytes / 16;  // 16-byte chunks per token row
  constexpr int kBlockBytes = 128 * 128;
  for (int idx = lane; idx < nrows * kChunks; idx += 32) {
    const int r = r0 + idx / kChunks, cc = idx % kChunks;
    const int tok = t0 + (r - r0);
    uint4 val = make_uint4(0u, 0u, 0u, 0u);
    if (tok < N) {
      const int rk = tok / nl, n = tok - rk * nl;
      const int64_t off = ((static_cast<int64_t>(rk) * B + b) * nl + n) * H * kRowBytes +
                          static_cast<int64_t>(head) * kRowBytes + cc * 16;
      val = kCoherent ? ld_global_v4(base + off) : ld_global_nc_v4(base + off);
    }
    st_shared_v4(dst + (cc >> 3) * kBlockBytes + r * 128 + (((cc & 7) ^ (r & 7)) << 4), val);
  }
  fence_proxy_async_smem();
}

// The kernel body.  kPeer: Q tiles come from the ranks' shards through
// `peer` (tmQ unused) and O rows go to the ranks' output shards; K and V are
// this rank's received head group, addressed as for the fused call.
// kSparse: a block mask over 64-token cubes restricts which keys each query
// attends.  Each query tile walks only the key cubes that one of its two
// query cubes selects, two cubes per 128-key step, from a per-CTA plan
// listing first the cubes both tiles visit; where both walks are at the same
// pair, one K/V load serves both.  Each row masks the cubes its own query
// cube did not select.
template <int D, bool kF8, bool kPeer, bool kSparse = false>
__device__ __forceinline__ void attention_body(const CUtensorMap *tmQ, const CUtensorMap *tmK,
                                               const CUtensorMap *tmV, const AttnParams &p,
                                               const PeerArgs *peer) {
  using C = AttnCfg<D, kF8>;
  static_assert(!kSparse || C::kHalves == 2, "the block-sparse loads take two column blocks");
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t *sptr = smem_raw + (sbase - raw);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int hg = blockIdx.y;            // global head
  const int b = blockIdx.z;
  const int map_head = hg % p.hsplit;
  const int map_batch = (hg / p.hsplit) * p.B + b;
  const int q0 = blockIdx.x * 2 * C::kBM;
  const int T = p.num_kv_tiles;

  const uint32_t bar_q = sbase + C::kOffBar;
  const uint32_t bar_kv_full = bar_q + 8;
  const uint32_t bar_kv_empty = bar_kv_full + 8 * C::kStages;
  const uint32_t bar_s = bar_kv_empty + 8 * C::kStages;  // [2]
  const uint32_t bar_p = bar_s + 16;                      // [2 tiles][2 key halves]
  const uint32_t bar_o = bar_p + 32;                      // [2]
  const uint32_t bar_drain = bar_o + 16;                  // the MMA thread's last commit
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sptr + C::kOffMisc);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(sptr + C::kOffMisc + 4);
  int *slot_item = reinterpret_cast<int *>(sptr + C::kOffMisc + 16);
  int *plan_n = reinterpret_cast<int *>(sptr + C::kOffCount);
  uint16_t *plan = reinterpret_cast<uint16_t *>(sptr + C::kOffPlan);
  const int64_t mask_row0 = (static_cast<int64_t>(b) * p.H + hg) * p.ncube;
  if constexpr (kSparse) {
    // The plan, built once per CTA by warps 0 and 1.  Query tile t (query
    // cubes 4x + 2t and 4x + 2t + 1) visits the key cubes either of them
    // selects: first those the other tile visits too, then its own, each
    // group in increasing order, two per 128-key step.  Both tiles' walks
    // then start with the same pairs, which one K/V load serves; the rest of
    // the steps take a load per tile.  Bits past the last cube are ignored.
    if (warp < 2) {
      const int t = warp;
      const int qa = blockIdx.x * 4;
      uint16_t *list = plan + t * C::kPlanStride;
      int n = 0;
      for (int pass = 0; pass < 2; ++pass) {
        for (int w0 = 0; w0 < p.nwords; w0 += 32) {
          const int w = w0 + lane;
          uint32_t bits = 0u;
          if (w < p.nwords) {
            uint32_t u0 = 0u, u1 = 0u;
            for (int qc = qa; qc < qa + 4 && qc < p.ncube; ++qc) {
              const uint32_t row = __ldg(p.mask + (mask_row0 + qc) * p.nwords + w);
              if (qc < qa + 2) u0 |= row;
              else u1 |= row;
            }
            if (w == p.nwords - 1 && (p.ncube & 31)) {
              u0 &= (1u << (p.ncube & 31)) - 1u;
              u1 &= (1u << (p.ncube & 31)) - 1u;
            }
            bits = pass == 0 ? (u0 & u1) : t == 0 ? (u0 & ~u1) : (u1 & ~u0);
          }
          // exclusive prefix of the lanes' counts: where this lane's cubes go
          const int cnt = __popc(bits);
          int incl = cnt;
#pragma unroll
          for (int d = 1; d < 32; d <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, d);
            if (lane >= d) incl += v;
          }
          int pos = n + incl - cnt;
          while (bits != 0u) {
            list[pos++] = static_cast<uint16_t>(32 * w + __ffs(bits) - 1);
            bits &= bits - 1u;
          }
          n += __shfl_sync(0xffffffffu, incl, 31);
        }
      }
      if (lane == 0) {
        if (n & 1) list[n] = static_cast<uint16_t>(p.ncube);
        plan_n[t] = n;
      }
    }
  }
  // Step i of tile t's walk: cubes (x, y) = list entries 2i and 2i + 1
  // (y = ncube: zero rows); the walk has ceil(n_t / 2) steps.
  auto pair_at = [&](int t, int i) -> int2 {
    const uint32_t v = *reinterpret_cast<const uint32_t *>(plan + t * C::kPlanStride + 2 * i);
    return make_int2(static_cast<int>(v & 0xffffu), static_cast<int>(v >> 16));
  };

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(bar_kv_full + 8 * s, 1);
      mbar_init(bar_kv_empty + 8 * s, 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar_s + 8 * t, 1);
      mbar_init(bar_p + 16 * t, 128);
      mbar_init(bar_p + 16 * t + 8, 128);
      mbar_init(bar_o + 8 * t, 1);
    }
    mbar_init(bar_drain, 1);
    *abort_flag = 0;
    for (int s = 0; s < C::kStages; ++s) slot_item[s] = -1;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(smem_u32(tmem_slot), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  bool ok = true;
  bool q_issued = false;  // the Q copies were issued (producer warp 8)
  // Block-sparse kernel: 12 warps, so that its per-row mask state fits.  The
  // third warpgroup (two TMA producers, the MMA warp and an idle warp) gives
  // registers to the two softmax warpgroups: 384 x 168 at launch =
  // 2 x 128 x 208 + 128 x 88, and each sub-partition holds 208 + 208 + 88
  // registers per lane (<= 512).
  constexpr bool kSplitRegs = kSparse;
  if (warp == 8 || (kSparse && warp == 10)) {
    if constexpr (kSplitRegs) asm volatile("setmaxnreg.dec.sync.aligned.u32 88;");
    // ---------------------------------------------------------------- producer
    // Warp 8 loads Q and the K/V ring; in the block-sparse kernel warp 10
    // loads the ring's V slots and warp 8 its K slots, since each slot there
    // takes four TMA boxes (two cubes x two 128-byte column blocks), which
    // four lanes issue together.  Otherwise one elected lane issues the TMA
    // loads.  In the rank-major layout a
    // 128-token tile that crosses a shard boundary is two strided blocks,
    // which one TMA box cannot describe: the whole warp copies such a tile
    // with 16-byte loads into the same 128-byte-swizzled layout the TMA
    // writes (16-byte chunk c of row r at chunk c ^ (r mod 8)), fences the
    // generic-proxy writes for the async proxy, and arrives without bytes.
    const uint64_t pol_q = policy_evict_first();
    const uint64_t pol_kv = policy_evict_last();
    if (lane == 0) {
      if (!kPeer) prefetch_tmap(tmQ);
      prefetch_tmap(tmK);
      prefetch_tmap(tmV);
    }
    const int nl = p.nl_split;
    auto tma_ok = [&](int t0) {
      if (nl == 0) return true;
      const int r0 = t0 / nl;
      return t0 - r0 * nl + C::kBM <= nl;
    };
    auto tma_tile = [&](const CUtensorMap *m, uint32_t dst, uint32_t bar, int t0, uint64_t pol) {
      if (nl == 0) {
        for (int h = 0; h < C::kHalves; ++h)
          tma_load_4d(dst + h * C::kBlockBytes, m, bar, h * C::kBoxInner, map_head, t0, map_batch,
                      pol);
      } else {
        const int r0 = t0 / nl;
        for (int h = 0; h < C::kHalves; ++h)
          tma_load_5d(dst + h * C::kBlockBytes, m, bar, h * C::kBoxInner, map_head, t0 - r0 * nl,
                      b, r0, pol);
      }
    };
    auto copy_tile = [&](const uint8_t *base, uint32_t dst, int t0, int r0 = 0,
                         int nrows = C::kBM) {
      copy_rows<C::kRowBytes, kPeer>(base, dst, t0, r0, nrows, p.N, nl, p.B, b, p.H, map_head, lane);
    };
    // Overlapped peer step: before the first load of tokens t0 .. t1, lane 0
    // waits (bounded) until the chunk of every rank holding one of them has
    // arrived, then orders its later TMA loads after that observation; the
    // other lanes' loads follow through __shfl_sync.  `arrived` (lane 0 only)
    // keeps the ranks already seen.
    uint32_t arrived = 0u;
    auto await_tokens = [&](int t0, int t1) -> bool {
      if (!kPeer || p.counts == nullptr) return true;
      bool good = true;
      if (lane == 0) {
        const int last = t1 < p.N - 1 ? t1 : p.N - 1;
        for (int r = t0 / p.count_nl; t0 <= last && r <= last / p.count_nl && good; ++r) {
          if ((arrived >> r) & 1u) continue;
          good = wait_counter_geq(p.counts + r, p.count_target, abort_flag, p.count_wait_ns);
          if (good) arrived |= 1u << r;
        }
        if (good) fence_proxy_async_global();
      }
      return __shfl_sync(0xffffffffu, good ? 1 : 0, 0) != 0;
    };
    // Peer Q: a tile inside one rank's shard is one TMA box per column block
    // from that rank's map; a tile that crosses ranks is gathered row by row.
    auto peer_q_ok = [&](int t0) {
      const int r0 = t0 / peer->nl;
      return r0 < peer->nranks && t0 - r0 * peer->nl + C::kBM <= peer->nl;
    };
    auto copy_q_peer = [&](uint32_t dst, int t0) {
      constexpr int kChunks = C::kRowBytes / 16;
      const int pnl = peer->nl;
      for (int idx = lane; idx < C::kBM * kChunks; idx += 32) {
        const int r = idx / kChunks, cc = idx % kChunks;
        const int tok = t0 + r;
        uint4 val = make_uint4(0u, 0u, 0u, 0u);
        if (tok < p.N) {
          const int rk = tok / pnl, n = tok - rk * pnl;
          const int64_t off = ((static_cast<int64_t>(b) * pnl + n) * peer->heads +
                               peer->head0 + hg) * C::kRowBytes + cc * 16;
          val = ld_global_v4(peer->q_ptr[rk] + off);
        }
        st_shared_v4(dst + (cc >> 3) * C::kBlockBytes + r * 128 + (((cc & 7) ^ (r & 7)) << 4), val);
      }
      fence_proxy_async_smem();
    };
    // Q: both tiles complete one barrier.
    const bool q_loader = warp == 8;
    ok = !q_loader || await_tokens(q0, q0 + 2 * C::kBM - 1);
    uint32_t q_tx = 0;
    for (int t = 0; t < 2 && ok && q_loader; ++t) {
      const uint32_t dst = sbase + C::kOffQ + t * C::kTileBytes;
      if (kPeer) {
        if (peer_q_ok(q0 + t * C::kBM)) q_tx += C::kTileBytes;
        else copy_q_peer(dst, q0 + t * C::kBM);
      } else {
        if (tma_ok(q0 + t * C::kBM)) q_tx += C::kTileBytes;
        else copy_tile(p.q, dst, q0 + t * C::kBM);
      }
    }
    __syncwarp();
    q_issued = ok && q_loader;
    if (lane == 0 && q_issued) {
      mbar_arrive_expect_tx(bar_q, q_tx);
      for (int t = 0; t < 2; ++t) {
        const int t0 = q0 + t * C::kBM;
        const uint32_t dst = sbase + C::kOffQ + t * C::kTileBytes;
        if (kPeer) {
          if (peer_q_ok(t0)) {
            const int r0 = t0 / peer->nl;
            for (int h = 0; h < C::kHalves; ++h)
              tma_load_4d(dst + h * C::kBlockBytes, &peer->q[r0], bar_q, h * C::kBoxInner,
                          peer->head0 + hg, t0 - r0 * peer->nl, b, pol_q);
          }
        } else if (tma_ok(t0)) {
          tma_tile(tmQ, dst, bar_q, t0, pol_q);
        }
      }
    }
    // Block-sparse: column block h of the 64 rows of the cube starting at
    // token t0, one TMA box (the maps' boxes are 64 rows); a row coordinate
    // at or past N reads zeros.
    auto tma_box = [&](const CUtensorMap *m, uint32_t d, uint32_t bar, int h, int t0) {
      if (nl == 0) {
        tma_load_4d(d, m, bar, h * C::kBoxInner, map_head, t0, map_batch, pol_kv);
      } else {
        const int r = t0 / nl;
        tma_load_5d(d, m, bar, h * C::kBoxInner, map_head, t0 - r * nl, b, r, pol_kv);
      }
    };
    auto tma_cube_ok = [&](int t0) {
      if (nl == 0) return true;
      const int r = t0 / nl;
      return t0 - r * nl + 64 <= nl;
    };
    int it = 0;
    if constexpr (!kSparse) {
      for (int j = 0; j < T && ok; ++j) {
        if (!await_tokens(j * C::kBN, j * C::kBN + C::kBN - 1)) {
          ok = false;
          break;
        }
        for (int kv = 0; kv < 2; ++kv, ++it) {
          const int s = it % C::kStages;
          const uint32_t ph = (it / C::kStages) & 1;
          const bool free_slot = mbar_wait(bar_kv_empty + 8 * s, ph ^ 1u, abort_flag, kWaitLimitNs);
          if (!__all_sync(0xffffffffu, free_slot)) {
            ok = false;
            break;
          }
          const uint32_t dst = sbase + C::kOffKV + s * C::kTileBytes;
          const uint32_t bar = bar_kv_full + 8 * s;
          if (lane == 0) slot_item[s] = it;
          if (tma_ok(j * C::kBN)) {
            if (lane == 0) {
              mbar_arrive_expect_tx(bar, C::kTileBytes);
              tma_tile(kv == 0 ? tmK : tmV, dst, bar, j * C::kBN, pol_kv);
            }
          } else {
            copy_tile(kv == 0 ? p.k : p.v, dst, j * C::kBN);
            __syncwarp();
            if (lane == 0) mbar_arrive(bar);
          }
          __syncwarp();
        }
      }
    } else {
      // Ring position it: K (kv = 0) or V (kv = 1) rows of the cube pair pr,
      // cube pr.x in rows 0..63 and cube pr.y (zeros when ncube) in 64..127.
      // Each warp loads the positions of its own kind and steps over the rest.
      const int my_kv = warp == 8 ? 0 : 1;
      auto load_pair = [&](int kv, int2 pr) -> bool {
        const int pos = it++;
        if (kv != my_kv) return true;
        const int s = pos % C::kStages;
        const uint32_t ph = (pos / C::kStages) & 1;
        const bool free_slot = mbar_wait(bar_kv_empty + 8 * s, ph ^ 1u, abort_flag, kWaitLimitNs);
        if (!__all_sync(0xffffffffu, free_slot)) return false;
        const uint32_t dst = sbase + C::kOffKV + s * C::kTileBytes;
        const uint32_t bar = bar_kv_full + 8 * s;
        const int t0 = 64 * pr.x, t1 = 64 * pr.y;
        const bool tma0 = tma_cube_ok(t0);
        const bool tma1 = pr.y < p.ncube ? tma_cube_ok(t1) : nl == 0;
        const uint8_t *src = kv == 0 ? p.k : p.v;
        // one copy loop for both halves (the producer runs on 88 registers)
        for (int hf = 0; hf < 2; ++hf)
          if (!(hf ? tma1 : tma0)) copy_tile(src, dst, hf ? t1 : t0, 64 * hf, 64);
        __syncwarp();
        if (lane == 0) {
          slot_item[s] = pos;
          mbar_arrive_expect_tx(bar, (tma0 ? C::kTileBytes / 2 : 0) + (tma1 ? C::kTileBytes / 2 : 0));
        }
        __syncwarp();
        // lane 2 hf + h copies cube half hf, column block h: one TMA box each
        if (lane < 2 * C::kHalves && ((lane >> 1) ? tma1 : tma0))
          tma_box(kv == 0 ? tmK : tmV, dst + (lane & 1) * C::kBlockBytes + (lane >> 1) * 64 * 128,
                  bar, lane & 1, (lane >> 1) ? t1 : t0);
        __syncwarp();
        return true;
      };
      // The ring order, which the MMA thread follows: K of both walks' first
      // steps, then per step i the V of step i and K of step i+1 for query
      // tile 0, then the same for tile 1; a slot is loaded once when both
      // walks are at the same pair.
      const int len0 = plan_n[0], len1 = plan_n[1];
      bool a0 = len0 > 0, a1 = len1 > 0;
      int2 c0 = a0 ? pair_at(0, 0) : make_int2(0, 0), c1 = a1 ? pair_at(1, 0) : make_int2(0, 0);
      if (ok && a0) ok = load_pair(0, c0);
      if (ok && a1 && !(a0 && c0.x == c1.x && c0.y == c1.y)) ok = load_pair(0, c1);
      for (int i = 1; ok && (a0 || a1); ++i) {
        const bool na0 = 2 * i < len0, na1 = 2 * i < len1;
        const int2 n0 = na0 ? pair_at(0, i) : c0, n1 = na1 ? pair_at(1, i) : c1;
        const bool sh_cur = a0 && a1 && c0.x == c1.x && c0.y == c1.y;
        const bool sh_nxt = na0 && na1 && n0.x == n1.x && n0.y == n1.y;
        if (a0) ok = load_pair(1, c0) && (!na0 || load_pair(0, n0));
        if (ok && a1 && !sh_cur) ok = load_pair(1, c1);
        if (ok && na1 && !sh_nxt) ok = load_pair(0, n1);
        c0 = n0;
        c1 = n1;
        a0 = na0;
        a1 = na1;
      }
    }
  } else if (warp == 9) {
    if constexpr (kSplitRegs) asm volatile("setmaxnreg.dec.sync.aligned.u32 88;");
    // ---------------------------------------------------------------- MMA issue
    if (lane == 0) {
      constexpr uint32_t idesc_qk = kF8 ? make_idesc_e4m3(128, 128, 0, 0)
                                        : make_idesc_bf16(128, 128, 0, 0);
      constexpr uint32_t idesc_pv = kF8 ? make_idesc_e4m3(128, D, 0, 1)
                                        : make_idesc_bf16(128, D, 0, 1);
      // Shared-memory descriptors are built once; an operand's start address
      // lives in the low 14 bits (address >> 4), so moving to another tile,
      // slot or K step is one integer add (all addresses stay below 256 KB).
      // This keeps the issuing thread far below the tensor core's 64 cycles
      // per 128 x 128 x 16 MMA although it shares its SM sub-partition with
      // two softmax warps.
      const uint64_t dQ = make_sdesc_sw128(sbase + C::kOffQ, 16, 1024);
      const uint64_t dK = make_sdesc_sw128(sbase + C::kOffKV, 16, 1024);
      const uint64_t dV = make_sdesc_sw128(sbase + C::kOffKV, C::kBlockBytes, 1024);
      auto issue_s = [&](int t, int slot) {
        const uint64_t a0 = dQ + static_cast<uint32_t>((t * C::kTileBytes) >> 4);
        const uint64_t b0 = dK + static_cast<uint32_t>((slot * C::kTileBytes) >> 4);
        const uint32_t d = tmem + (t ? C::kColS1 : 0u);
#pragma unroll
        for (int kk = 0; kk < C::kQkSteps; ++kk) {
          const uint32_t off = ((kk >> 2) * C::kBlockBytes + (kk & 3) * 32) >> 4;
          umma_ss<kF8>(d, a0 + off, b0 + off, idesc_qk, kk > 0 ? 1u : 0u);
        }
      };
      // O_t += P_t[:, 64h .. 64h+63] V_j[64h .. 64h+63, :] for key half h.
      auto issue_pv_half = [&](int t, int slot, bool first, int h) {
        const uint64_t b0 = dV + static_cast<uint32_t>((slot * C::kTileBytes) >> 4);
        const uint32_t a0 = tmem + (t ? C::kColS1 : 0u);
        const uint32_t d = tmem + (t ? C::kColO1 : C::kColO0);
#pragma unroll
        for (int k = 0; k < C::kPvSteps / 2; ++k) {
          const int kk = (C::kPvSteps / 2) * h + k;
          umma_ts<kF8>(d, a0 + kk * 8, b0 + static_cast<uint32_t>((kk * C::kPvKeys * 128) >> 4),
                       idesc_pv, (first && kk == 0) ? 0u : 1u);
        }
      };
      // Waits for each half of P_t, then issues that half's PV MMAs.
      auto issue_pv = [&](int t, int slot, bool first, int j) -> bool {
        for (int h = 0; h < 2; ++h) {
          if (!mbar_wait(bar_p + 16 * t + 8 * h, j & 1, abort_flag, kWaitLimitNs)) return false;
          tc_fence_after();
          issue_pv_half(t, slot, first, h);
        }
        return true;
      };
      int it = 0;
      // Q has landed before anything else happens (also when no key tile is
      // selected, so that no copy into shared memory outlives the CTA).
      ok = mbar_wait(bar_q, 0, abort_flag, kWaitLimitNs);
      if constexpr (!kSparse) {
        ok = ok && mbar_wait(bar_kv_full, 0, abort_flag, kWaitLimitNs);
        if (ok) {
          tc_fence_after();
          issue_s(0, 0);
          umma_commit(bar_s);
          issue_s(1, 0);
          umma_commit(bar_s + 8);
          umma_commit(bar_kv_empty);
          it = 1;
        }
        for (int j = 0; j < T && ok; ++j) {
          const bool more = j + 1 < T;
          // Both K/V waits come first: the loads landed long ago, and no
          // barrier wait sits between a tile's PV and its next S.
          const int sv = it % C::kStages;
          ok = mbar_wait(bar_kv_full + 8 * sv, (it / C::kStages) & 1, abort_flag, kWaitLimitNs);
          ++it;
          if (!ok) break;
          int sk = 0;
          if (more) {
            sk = it % C::kStages;
            ok = mbar_wait(bar_kv_full + 8 * sk, (it / C::kStages) & 1, abort_flag, kWaitLimitNs);
            ++it;
            if (!ok) break;
          }
          ok = issue_pv(0, sv, j == 0, j);
          if (!ok) break;
          if (more) {
            issue_s(0, sk);
            umma_commit(bar_s);
          } else {
            umma_commit(bar_o);
          }
          ok = issue_pv(1, sv, j == 0, j);
          if (!ok) break;
          if (more) {
            issue_s(1, sk);
            umma_commit(bar_s + 8);
            umma_commit(bar_kv_empty + 8 * sv);
            umma_commit(bar_kv_empty + 8 * sk);
          } else {
            umma_commit(bar_o + 8);
            umma_commit(bar_kv_empty + 8 * sv);
          }
        }
      } else {
        // Each query tile walks its own cube pairs, in the producer's ring
        // order.  Per step i: O_0 += P_0 V_0(i), S_0 = Q_0 K_0(i+1)^T, then
        // the same for tile 1; a slot shared by both walks is released after
        // tile 1's MMAs, any other one after its own tile's.  A tile whose
        // walk is shorter stops early: its O barrier follows its last PV, and
        // a tile with no selected cube commits it before any MMA (its rows
        // come out as zeros).
        auto take = [&](int &slot) -> bool {
          slot = it % C::kStages;
          const bool got =
              mbar_wait(bar_kv_full + 8 * slot, (it / C::kStages) & 1, abort_flag, kWaitLimitNs);
          ++it;
          return got;
        };
        const int len0 = plan_n[0], len1 = plan_n[1];
        bool a0 = len0 > 0, a1 = len1 > 0;
        int2 c0 = a0 ? pair_at(0, 0) : make_int2(0, 0), c1 = a1 ? pair_at(1, 0) : make_int2(0, 0);
        if (ok && !a0) umma_commit(bar_o);
        if (ok && !a1) umma_commit(bar_o + 8);
        const bool sh0 = a0 && a1 && c0.x == c1.x && c0.y == c1.y;
        int sk0 = 0, sk1 = 0;
        if (ok && a0) {
          ok = take(sk0);
          if (ok) {
            tc_fence_after();
            issue_s(0, sk0);
            umma_commit(bar_s);
            if (!sh0) umma_commit(bar_kv_empty + 8 * sk0);
          }
        }
        if (ok && a1) {
          if (sh0) sk1 = sk0;
          else ok = take(sk1);
          if (ok) {
            tc_fence_after();
            issue_s(1, sk1);
            umma_commit(bar_s + 8);
            umma_commit(bar_kv_empty + 8 * sk1);
          }
        }
        for (int jj = 0; ok && (a0 || a1); ++jj) {
          const bool na0 = 2 * (jj + 1) < len0, na1 = 2 * (jj + 1) < len1;
          const int2 n0 = na0 ? pair_at(0, jj + 1) : c0, n1 = na1 ? pair_at(1, jj + 1) : c1;
          const bool sh_cur = a0 && a1 && c0.x == c1.x && c0.y == c1.y;
          const bool sh_nxt = na0 && na1 && n0.x == n1.x && n0.y == n1.y;
          int sv0 = 0;
          sk0 = 0;
          if (a0) {
            ok = take(sv0) && (!na0 || take(sk0));
            ok = ok && issue_pv(0, sv0, jj == 0, jj);
            if (!ok) break;
            if (na0) {
              issue_s(0, sk0);
              umma_commit(bar_s);
            } else {
              umma_commit(bar_o);
            }
            if (!sh_cur) umma_commit(bar_kv_empty + 8 * sv0);
            if (na0 && !sh_nxt) umma_commit(bar_kv_empty + 8 * sk0);
          }
          if (a1) {
            int sv1 = sv0;
            sk1 = sk0;
            if (!sh_cur) ok = take(sv1);
            if (ok && na1 && !sh_nxt) ok = take(sk1);
            ok = ok && issue_pv(1, sv1, jj == 0, jj);
            if (!ok) break;
            if (na1) {
              issue_s(1, sk1);
              umma_commit(bar_s + 8);
            } else {
              umma_commit(bar_o + 8);
            }
            umma_commit(bar_kv_empty + 8 * sv1);
            if (na1) umma_commit(bar_kv_empty + 8 * sk1);
          }
          c0 = n0;
          c1 = n1;
          a0 = na0;
          a1 = na1;
        }
      }
    }
    __syncwarp();
  } else if (kSplitRegs && warp >= 10) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 88;");  // idle: registers to the softmax
  } else {
    if constexpr (kSplitRegs) asm volatile("setmaxnreg.inc.sync.aligned.u32 208;");
    // ---------------------------------------------------------------- softmax
    const int t = warp >> 2;           // query tile
    const int wq = warp & 3;           // TMEM lane quarter this warp may access
    const int row = wq * 32 + lane;    // row within the tile
    const uint32_t lane_bits = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tS = tmem + lane_bits + (t ? C::kColS1 : 0u);
    const uint32_t tO = tmem + lane_bits + (t ? C::kColO1 : C::kColO0);
    // E4M3: the logits carry the factor of this query tile's token block
    // and, per key tile j, the factor of key block j (read one step ahead).
    const int bh = b * p.H + hg;
    const int qblk = blockIdx.x * 2 + t;
    const float sl2q = kF8 && qblk < p.nblk ? p.scale_log2e * p.dq[bh * p.nblk + qblk]
                                            : p.scale_log2e;
    const float *dk_row = kF8 ? p.dk + static_cast<int64_t>(bh) * p.nblk : nullptr;
    float dk_next = kF8 ? __ldg(dk_row) : 1.0f;
    const int tail = p.N - (T - 1) * C::kBN;   // valid keys in the last tile, 1..128
    float m_ref = -INFINITY;                   // reference maximum, log2 units
    float l = 0.f;
    // Block-sparse variant: this row's mask words (its 64-token query cube);
    // rows past the last cube select nothing.
    const int qcube = (q0 + t * C::kBM + row) >> 6;
    const uint32_t *mrow = kSparse && qcube < p.ncube ? p.mask + (mask_row0 + qcube) * p.nwords
                                                     : nullptr;
    // Sparse: this tile's walk; step jj covers cubes pr.x (keys 0..63) and
    // pr.y (keys 64..127, ncube when none).  Dense: step jj is key tile jj.
    const int steps = kSparse ? (plan_n[t] + 1) / 2 : T;
    for (int jj = 0; jj < steps; ++jj) {
      const int2 pr = kSparse ? pair_at(t, jj) : make_int2(jj, 0);
      const int j = pr.x;
      [[maybe_unused]] const int cb = pr.y;
      // Warp-uniform exit: the TMEM accesses below are warp-collective.
      const bool got = mbar_wait(bar_s + 8 * t, jj & 1, abort_flag, kWaitLimitNs);
      if (!__all_sync(0xffffffffu, got)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const float sl2 = kF8 ? sl2q * dk_next : sl2q;
      if (kF8 && j + 1 < T) dk_next = __ldg(dk_row + j + 1);
      uint32_t s[128];
      tmem_ld32(tS + 0, &s[0]);
      tmem_ld32(tS + 32, &s[32]);
      tmem_ld32(tS + 64, &s[64]);
      tmem_ld32(tS + 96, &s[96]);
      tmem_wait_ld();
      if constexpr (!kSparse) {
        if (j == T - 1 && tail < C::kBN) {
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (c >= tail) s[c] = 0xFF800000u;  // -inf
        }
      } else {
        // keys at or past N (zero rows in shared memory) of a partial last
        // cube (key cubes are 0 .. ncube-1)
        const int lim0 = j == p.ncube - 1 ? p.N - 64 * j : 64;
        const int lim1 = cb == p.ncube - 1 ? p.N - 64 * cb : 64;
        if (lim0 < 64 || lim1 < 64) {
#pragma unroll
          for (int c = 0; c < 64; ++c) {
            if (c >= lim0) s[c] = 0xFF800000u;
            if (c >= lim1) s[64 + c] = 0xFF800000u;
          }
        }
      }
      // Row maximum: eight independent chains of 3-input max over 16
      // scores each, then a short tree.
      float mc[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const uint32_t *e = &s[16 * q];
        float m = fmax3(__uint_as_float(e[0]), __uint_as_float(e[1]), __uint_as_float(e[2]));
#pragma unroll
        for (int c = 3; c < 15; c += 2)
          m = fmax3(m, __uint_as_float(e[c]), __uint_as_float(e[c + 1]));
        mc[q] = fmaxf(m, __uint_as_float(e[15]));
      }
      // Sparse: cube j is the tile's first half, cube cb its second; a half
      // this row's query cube did not select counts for neither the maximum
      // nor the sum.
      bool sel0 = true, sel1 = true;
      if constexpr (kSparse) {
        sel0 = mrow != nullptr && ((__ldg(mrow + (j >> 5)) >> (j & 31)) & 1u) != 0u;
        sel1 = mrow != nullptr && cb < p.ncube && ((__ldg(mrow + (cb >> 5)) >> (cb & 31)) & 1u) != 0u;
      }
      float mx;
      if constexpr (kSparse) {
        const float h0 = fmaxf(fmax3(mc[0], mc[1], mc[2]), mc[3]);
        const float h1 = fmaxf(fmax3(mc[4], mc[5], mc[6]), mc[7]);
        mx = fmaxf(sel0 ? h0 : -INFINITY, sel1 ? h1 : -INFINITY) * sl2;
      } else {
        mx = fmax3(fmax3(mc[0], mc[1], mc[2]), fmax3(mc[3], mc[4], mc[5]),
                   fmaxf(mc[6], mc[7])) * sl2;
      }
      const bool need = mx > m_ref + C::kThresh;
      const bool warp_rescale = __any_sync(0xffffffffu, need);
      const float alpha = need ? ex2(m_ref - mx) : 1.0f;
      if (need) {
        l *= alpha;
        m_ref = mx;
      }
      // p = 2^(s * scale * log2(e) - m_ref): two scores per packed FMA, ex2
      // on the SFU.  Each half of the row's 128 probabilities is stored to TMEM
      // (bf16, over the first 64 columns of S_t) and signalled on its own, so
      // the PV MMAs of keys 0..63 can start while keys 64..127 are computed.
      const uint64_t k_sl2 = f2_pack(sl2, sl2);
      const uint64_t k_negm = f2_pack(C::kShift - m_ref, C::kShift - m_ref);
      // Sparse: an unselected half gets a bias of -inf (its probabilities are
      // 0); a row that has not met a selected key yet keeps m = -inf and uses
      // a bias of 0 for its (then all -inf) scores.
      float bias_h[2] = {0.f, 0.f};
      if constexpr (kSparse) {
        const float bias = C::kShift - (m_ref > -INFINITY ? m_ref : 0.f);
        bias_h[0] = sel0 ? bias : -INFINITY;
        bias_h[1] = sel1 ? bias : -INFINITY;
      }
      uint64_t acc[2] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint64_t k_bias = kSparse ? f2_pack(bias_h[h], bias_h[h]) : k_negm;
        uint32_t pk[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const int c = 64 * h + 2 * i;
          const uint64_t x = f2_fma(f2_pack_bits(s[c], s[c + 1]), k_sl2, k_bias);
          float p0, p1;
          f2_unpack(x, p0, p1);
          p0 = ex2(p0);
          p1 = ex2(p1);
          acc[i & 1] = f2_add(acc[i & 1], f2_pack(p0, p1));
          if (kF8) {
            // four E4M3 probabilities per 32-bit column, key order in bytes
            const uint32_t two = pack_e4m3x2(p0, p1);
            pk[i >> 1] = (i & 1) ? (pk[i >> 1] | (two << 16)) : two;
          } else {
            pk[i] = pack_bf16x2(p0, p1);
          }
        }
        if (h == 0 && warp_rescale && jj > 0) {
          // Rescale O_t by alpha before any PV MMA of this tile (warp-uniform
          // because TMEM access is warp-collective; rows that keep their
          // reference multiply by exactly 1).  O_t is complete: the commit
          // that signalled S_t also covered the previous PV.
#pragma unroll 1
          for (int c = 0; c < D; c += 32) {
            uint32_t o[32];
            tmem_ld32(tO + c, o);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32(tO + c, o);
          }
        }
        if (kF8)
          tmem_st16(tS + (C::kPCols / 2) * h, pk);
        else
          tmem_st32(tS + (C::kPCols / 2) * h, pk);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar_p + 16 * t + 8 * h);
      }
      {
        float a0, a1, b0, b1;
        f2_unpack(acc[0], a0, a1);
        f2_unpack(acc[1], b0, b1);
        l += (a0 + a1) + (b0 + b1);
      }
    }
    // ------------------------------------------------------------ epilogue
    if (ok) ok = mbar_wait(bar_o + 8 * t, 0, abort_flag, kWaitLimitNs);
    if (__all_sync(0xffffffffu, ok)) {
      tc_fence_after();
      const int token = q0 + t * C::kBM + row;
      // Sparse: a row that attended no key (l = 0) is written as zeros.
      const bool valid = token < p.N && (!kSparse || l > 0.f);
      const bool exists = token < p.Np;
      const float inv_l = valid ? 1.0f / l : 0.0f;
      const float *dv_row = kF8 ? p.dv + static_cast<int64_t>(bh) * D : nullptr;
      int64_t row_off;
      __nv_bfloat16 *obase = p.o;
      int ohead = map_head;
      if (kPeer) {
        // this row belongs to rank token / nl; O goes straight to its shard
        const int rk = token / peer->nl, n = token - rk * peer->nl;
        obase = peer->o_ptr[rk < peer->nranks ? rk : 0];  // rows past Np are not stored
        row_off = (static_cast<int64_t>(b) * peer->nl + n) * peer->heads * D;
        ohead = peer->head0 + hg;
      } else if (p.nl_split) {
        const int rk = token / p.nl_split, n = token - rk * p.nl_split;
        row_off = static_cast<int64_t>(rk) * p.o_rank + static_cast<int64_t>(b) * p.o_batch +
                  static_cast<int64_t>(n) * p.o_row;
      } else {
        row_off = static_cast<int64_t>(map_batch) * p.o_batch + static_cast<int64_t>(token) * p.o_row;
      }
      __nv_bfloat16 *dst = obase + row_off + static_cast<int64_t>(ohead) * D;
#pragma unroll
      for (int c = 0; c < D; c += 32) {
        uint32_t o[32];
        tmem_ld32(tO + c, o);
        tmem_wait_ld();
        if (kF8) {
          // E4M3: channel c of O carries V's factor of channel c.
#pragma unroll
          for (int i = 0; i < 32; ++i)
            o[i] = __float_as_uint(__uint_as_float(o[i]) * __ldg(dv_row + c + i));
        }
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          w[i] = valid ? pack_bf16x2(__uint_as_float(o[2 * i]) * inv_l,
                                     __uint_as_float(o[2 * i + 1]) * inv_l)
                       : 0u;  // padding rows (and sparse rows with no key): +0.0 words
        if (exists) {
          uint4 *d4 = reinterpret_cast<uint4 *>(dst + c);
#pragma unroll
          for (int i = 0; i < 4; ++i)
            d4[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
        }
      }
      if (p.lse != nullptr && exists) {
        const float v = valid ? (m_ref - C::kShift + __log2f(l)) * 0.69314718055994531f
                              : -INFINITY;
        p.lse[(static_cast<int64_t>(b) * p.H + hg) * p.Np + token] = v;
      }
    } else {
      ok = false;
    }
  }

  // ------------------------------------------------------------------ teardown
  // Peer stores are ordered before whatever the host sequences after the
  // kernel (the end-of-step collective that lets the owners read O).
  if (kPeer) __threadfence_system();
  if (!ok) {
    *abort_flag = 1;
    atomicExch(p.status, kStatusTimeout);
  }
  tc_fence_before();
  __syncthreads();
  if (*abort_flag) {
    // Before the CTA's shared and tensor memory are released, let the
    // asynchronous work it issued land: the TMA copies of Q and of the last
    // load issued into each ring slot (earlier loads into a slot were
    // consumed, so they landed), and every MMA the issuing thread enqueued
    // (one more commit, then its barrier).  None of these depends on another
    // thread, so each bounded wait ends; if one does not, the status word
    // already holds the error.
    if (warp == 8 && lane == 0) {
      if (q_issued) mbar_wait_drain(bar_q, 0, kWaitLimitNs);
      for (int s = 0; s < C::kStages; ++s)
        if (slot_item[s] >= 0)
          mbar_wait_drain(bar_kv_full + 8 * s, (slot_item[s] / C::kStages) & 1, kWaitLimitNs);
    }
    if (warp == 9 && lane == 0) {
      umma_commit(bar_drain);
      mbar_wait_drain(bar_drain, 0, kWaitLimitNs);
    }
    __syncthreads();
  }
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

template <int D, bool kF8 = false>
__global__ void __launch_bounds__(320, 1)
attention_kernel(const __grid_constant__ CUtensorMap tmQ,
                 const __grid_constant__ CUtensorMap tmK,
                 const __grid_constant__ CUtensorMap tmV, const __grid_constant__ AttnParams p) {
  attention_body<D, kF8, false>(&tmQ, &tmK, &tmV, p, nullptr);
}

// Block-sparse attention (bf16, D = 128): the sequence-sharded fused call
// with a mask of selected 64-token key cubes per 64-token query cube.
__global__ void __launch_bounds__(384, 1)
attention_sparse_kernel(const __grid_constant__ CUtensorMap tmQ,
                        const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV,
                        const __grid_constant__ AttnParams p) {
  attention_body<128, false, false, true>(&tmQ, &tmK, &tmV, p, nullptr);
}

// One rank's step of the multi-GPU form (bf16, D = 128): Q read from every
// rank's shard and O written to every rank's output shard over peer
// addresses; K and V from this rank's received head group.
__global__ void __launch_bounds__(320, 1)
attention_peer_kernel(const __grid_constant__ PeerArgs peer,
                      const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const __grid_constant__ AttnParams p) {
  attention_body<128, false, true>(nullptr, &tmK, &tmV, p, &peer);
}

}  // namespace sp
