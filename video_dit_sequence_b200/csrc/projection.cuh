// projection.cuh -- the projections around attention as tcgen05 GEMMs whose
// operand loads or epilogue do the layout work of the Ulysses exchange.
//
// In front of attention (each token's hidden state to its q, k and v):
// y[m][c] = sum_k x[m][k] * w[c][k] (+ bias[c]) for the rows m of x and the
// 3*H*D output features c (q, then k, then v; a feature's weights are one row
// of w, as a linear layer stores them).  The pages never describe the
// transformer block around the attention, so no rotary embedding or
// normalisation is applied.  Feature c is element d of head h of tensor t
// (c = t*H*D + h*D + d); row m is a token of the sequence-sharded hidden
// states, and the epilogue stores y[m][c] at
//   kProjSeqSharded  [P][B][Nl][H][D]   (the fused attention's input),
//   kProjHeadSharded [P][B][Np][Hl][D]  (the pack folded in),
//   kProjSendChunks  [P][B][Nl][Hl][D]  (one rank's exchange pack folded in),
// so that no permutation pass runs between the projection and attention.
//
// After attention (the output projection y = o * w_o^T (+ bias), hidden
// features per token from the H*D attention outputs) the layout work moves
// to the operand side: the TMA loads of A read O where attention left it,
//   kALoadMatrix  [P][B][Nl][H][D]  sequence shards (the fused call's output)
//   kALoadHeads   [P][B][Np][Hl][D] head groups (sp_attention's output; the
//                 unpack folded in: a 64-wide K slice lies inside one head
//                 group, so it is one box of group j's rows)
//   kALoadChunks  [P][B][Nl][Hl][D] one rank's returned chunks (the exchange
//                 unpack folded in: K slice k lies in chunk k / (Hl*D))
// and the epilogue stores plain rows of y [P][B][Nl][hidden] (one rank's
// [B][Nl][hidden] for chunks).
//
// The GEMM runs on CTA pairs (a cluster of two CTAs on neighbouring SMs): a
// tile of y is 256 x 256, each CTA of the pair holds 128 of its rows of A
// and 128 of its rows of w (128-wide K slices through a 3-stage ring), and
// one thread of the even CTA issues 256 x 256 x 16 tcgen05 MMAs
// (cta_group::2) that read both CTAs' shared memory and accumulate each
// CTA's 128 rows in that CTA's tensor memory.  Against one CTA per 128 x 256
// tile, every SM moves a third less operand data per MMA.  A stage holds
// 128 elements of K (two boxes per operand; 3 stages of 64 KB).  Each CTA's loads
// complete on its own barrier; the odd CTA forwards that completion to the
// even one with a remote mbarrier arrive (no multicast; the plain arrive form,
// whose release is CTA-scoped: a cluster-scoped release per 512-cycle stage
// cost half the throughput).  Four epilogue warps
// per CTA (one per TMEM lane quarter) add the bias, round to bf16 and store
// 64-byte runs.  The kernel is persistent, one pair per two SMs, with two
// accumulators so that one tile's epilogue overlaps the next tile's MMAs;
// tiles run in groups of kProjGroupM row blocks so that the pairs working at
// one time share their x and w slices in L2.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "sm100.cuh"

namespace sp {

enum ProjLayout { kProjSeqSharded = 0, kProjHeadSharded = 1, kProjSendChunks = 2 };
// How the A operand's K slices are addressed (see the header comment).
enum ProjALoad { kALoadMatrix = 0, kALoadChunks = 1, kALoadHeads = 2 };

struct ProjParams {
  int32_t M, K, nout;        // rows of A, reduction size, output features
  int32_t H, D, Hl;          // heads, head dim, heads per group (H / P)
  int32_t P, B, Nl, Np;      // degree, batch, tokens per rank, P * Nl
  int32_t layout;            // ProjLayout (q, k, v projection)
  int32_t tiles_m, tiles_n;  // row blocks (all batch slots), column blocks
  __nv_bfloat16 *out[3];     // q, k, v
  const __nv_bfloat16 *bias; // [nout] or null
  int32_t *status;
  // Output projection (out_proj = 1): A read through a_load, y row-major.
  int32_t out_proj;
  int32_t a_load;            // ProjALoad
  int32_t a_cols;            // Hl*D: K columns of one head group / chunk
  int32_t rows_per_slot;     // A rows of one batch slot (Np for heads, else M)
  int32_t tiles_per_slot;    // row blocks of one batch slot
  __nv_bfloat16 *y;          // [rows][nout]
};

constexpr int kProjBN = 256;                      // features of a tile
constexpr int kProjBK = 64;                       // bf16 elements: one 128-byte row
constexpr int kProjGroupM = 16;
constexpr int kProjThreads = 192;                 // TMA, MMA, four epilogue warps
constexpr uint32_t kProjTmemCols = 512;           // two 256-column accumulators
constexpr uint64_t kProjWaitNs = 2000000000ull;   // 2 s per wait
constexpr int32_t kProjStatusTimeout = 7;         // SP_ERR_TIMEOUT

// A CTA pair per 256 x 256 tile (each CTA: 128 rows of A, 128 rows of w).  A
// stage holds 128 elements of K: two 64-wide boxes of each operand, so that
// every stage's barrier round trip and commit cover eight MMAs.
constexpr int kPairBM = 256;
constexpr int kPairStages = 3;
constexpr int kPairBoxes = 2;                     // 64-wide K boxes per operand per stage
constexpr int kPairBoxBytes = 128 * 128;          // 128 rows x 64 bf16: 16 KB
constexpr int kPairHalfBytes = kPairBoxes * kPairBoxBytes;   // one operand of a stage
constexpr int kPairStageBytes = 2 * kPairHalfBytes;
constexpr int kPairOffBar = kPairStages * kPairStageBytes;
constexpr int kPairOffMisc = kPairOffBar + (2 * kPairStages + 5) * 8;  // ..., bar_drain
constexpr int kPairSmemBytes = kPairOffMisc + 16 + 1024;

// Tile t of the y matrix as (row block, column block): groups of
// kProjGroupM row blocks, the column blocks of a group inside it.
__device__ __forceinline__ void proj_tile(int t, int tiles_m, int tiles_n, int &tm, int &tn) {
  const int per_group = kProjGroupM * tiles_n;
  const int g = t / per_group;
  const int first_m = g * kProjGroupM;
  const int gm = min(kProjGroupM, tiles_m - first_m);
  const int in_group = t - g * per_group;
  tm = first_m + in_group % gm;
  tn = in_group / gm;
}

// TMA loads of one 64-wide K slice of A: rows row0 .. row0 + box - 1 of batch
// slot `slot`, through the map built for p.a_load.
__device__ __forceinline__ void proj_load_a(const CUtensorMap *tmA, uint32_t dst, uint32_t bar,
                                            const ProjParams &p, int k0, int row0, int slot,
                                            uint64_t pol) {
  if (p.a_load == kALoadMatrix) {
    tma_load_4d(dst, tmA, bar, k0, row0, 0, 0, pol);
  } else {
    // a 64-wide K slice lies inside one head group (a_cols = Hl*D)
    const int grp = k0 / p.a_cols, c0 = k0 - grp * p.a_cols;
    if (p.a_load == kALoadChunks)
      tma_load_4d(dst, tmA, bar, c0, row0, grp, 0, pol);
    else
      tma_load_4d(dst, tmA, bar, c0, row0, slot, grp, pol);
  }
}

// Stores the 128 x 256 accumulator block in TMEM at taddr (this warp's lane
// quarter): lane `row` of the block is A row ar0 + row of batch slot `slot`,
// its features n0 .. n0 + 255.  `release()` runs once the whole block is in
// registers, so the MMAs may reuse the accumulator while the stores run.
template <typename Release>
__device__ __forceinline__ void proj_store_block(const ProjParams &p, uint32_t taddr, int slot,
                                                 int ar0, int n0, int row, int lane,
                                                 Release release) {
  const int ar = ar0 + row;
  if (p.out_proj) {
    // output projection: the y row of this token is its sequence-shard row
    int64_t yrow = -1;
    if (ar < p.rows_per_slot) {
      if (p.a_load == kALoadHeads) {  // token ar of batch slot `slot`
        const int r = ar / p.Nl, nn = ar - r * p.Nl;
        yrow = (static_cast<int64_t>(r) * p.B + slot) * p.Nl + nn;
      } else {
        yrow = ar;
      }
    }
    for (int c = 0; c < kProjBN; c += 32) {
      const int f = n0 + c;
      uint32_t accv[32];
      __syncwarp();                                     // TMEM loads are warp-collective
      tmem_ld32(taddr + c, accv);
      tmem_wait_ld();
      if (c + 32 == kProjBN) release();
      if (f >= p.nout || yrow < 0) continue;
      // nout is a multiple of 8: the chunk's last 16-byte vectors may lie
      // past the end of the row and are neither computed nor stored
      uint32_t w[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        float y0 = __uint_as_float(accv[2 * i]), y1 = __uint_as_float(accv[2 * i + 1]);
        if (p.bias != nullptr && f + 2 * i < p.nout) {
          y0 += __bfloat162float(p.bias[f + 2 * i]);
          y1 += __bfloat162float(p.bias[f + 2 * i + 1]);
        }
        w[i] = pack_bf16x2(y0, y1);
      }
      uint4 *dst = reinterpret_cast<uint4 *>(p.y + yrow * p.nout + f);
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (f + 8 * i < p.nout)
          dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
    }
    return;
  }
  // q, k, v projection (one batch slot: ar is the token row m of the
  // sequence-sharded hidden states); the row part of the destination offset
  // per layout
  const int m = ar;
  const int HD = p.H * p.D;
  int64_t row_seq = 0, row_head = 0;
  if (m < p.M) {
    row_seq = static_cast<int64_t>(m) * HD;
    if (p.layout == kProjHeadSharded) {
      const int bn = m % (p.B * p.Nl);                  // m = (r*B + b)*Nl + n
      const int r = m / (p.B * p.Nl), bb = bn / p.Nl, nn = bn - bb * p.Nl;
      row_head = static_cast<int64_t>(bb) * p.Np + static_cast<int64_t>(r) * p.Nl + nn;
    }
  }
  for (int c = 0; c < kProjBN; c += 32) {
    const int f = n0 + c;                               // first feature of the chunk
    uint32_t accv[32];
    __syncwarp();
    tmem_ld32(taddr + c, accv);
    tmem_wait_ld();
    if (c + 32 == kProjBN) release();
    if (f >= p.nout || m >= p.M) continue;              // after the collective load
    const int tt = f / HD, hd = f - tt * HD, h = hd / p.D, d = hd - h * p.D;
    int64_t off;
    if (p.layout == kProjSeqSharded) {
      off = row_seq + hd;
    } else {
      const int j = h / p.Hl, hh = h - j * p.Hl;
      const int64_t rows = p.layout == kProjHeadSharded
                               ? static_cast<int64_t>(j) * p.B * p.Np + row_head
                               : static_cast<int64_t>(j) * p.M + m;
      off = (rows * p.Hl + hh) * p.D + d;
    }
    uint32_t w[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      float y0 = __uint_as_float(accv[2 * i]), y1 = __uint_as_float(accv[2 * i + 1]);
      if (p.bias != nullptr) {
        y0 += __bfloat162float(p.bias[f + 2 * i]);
        y1 += __bfloat162float(p.bias[f + 2 * i + 1]);
      }
      w[i] = pack_bf16x2(y0, y1);
    }
    uint4 *dst = reinterpret_cast<uint4 *>(p.out[tt] + off);
#pragma unroll
    for (int i = 0; i < 4; ++i)
      dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
  }
}

// A CTA pair per 256 x 256 tile, launched as clusters of two CTAs.  Pair c
// (CTAs 2c and 2c + 1) computes tiles c, c + gridDim.x / 2, ...  CTA rank r
// holds A rows 128r .. 128r + 127 and w rows (features) 128r .. 128r + 127 of
// each tile, and the epilogue rows 128r .. 128r + 127 in its TMEM.
//   full[s]      rank 0: its own TMA bytes + one forwarded arrival from
//                rank 1 (rank 1's bytes landed); rank 1: its own TMA bytes
//   empty[s]     each rank: the MMA thread's commit after the stage's MMAs
//   acc_full[a]  each rank: the MMA thread's commit after a tile's MMAs
//   acc_empty[a] rank 0: one arrival per epilogue warp of both ranks
__global__ void __launch_bounds__(kProjThreads, 1)
projection_pair_kernel(const __grid_constant__ CUtensorMap tmX,
                       const __grid_constant__ CUtensorMap tmW, const __grid_constant__ ProjParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t *sptr = smem_raw + (sbase - raw);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int ntiles = p.tiles_m * p.tiles_n;
  // stages per tile; K slices past K read as zeros and add nothing
  const int nk = (p.K + kPairBoxes * kProjBK - 1) / (kPairBoxes * kProjBK);

  const uint32_t bar_full = sbase + kPairOffBar;                 // [stages]
  const uint32_t bar_empty = bar_full + 8 * kPairStages;          // [stages]
  const uint32_t bar_acc_full = bar_empty + 8 * kPairStages;      // [2]
  const uint32_t bar_acc_empty = bar_acc_full + 16;               // [2]
  const uint32_t bar_drain = bar_acc_empty + 16;                  // the MMA thread's last commit
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sptr + kPairOffMisc);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPairStages; ++s) {
      mbar_init(bar_full + 8 * s, rank == 0 ? 2 : 1);
      mbar_init(bar_empty + 8 * s, 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(bar_acc_full + 8 * a, 1);
      mbar_init(bar_acc_empty + 8 * a, 8);      // epilogue warps of both ranks (rank 0 only)
    }
    mbar_init(bar_drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), kProjTmemCols);
    tmem_relinquish_pair();
  }
  // both ranks' barriers are initialised and their TMEM allocated before
  // either rank signals the other
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  bool ok = true;
  int issued = 0;  // ring loads issued by the producer thread (abort-path drain)
  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      prefetch_tmap(&tmX);
      prefetch_tmap(&tmW);
      const uint64_t pol = policy_evict_last();
      int it = 0;
      for (int t = pair; t < ntiles && ok; t += npairs) {
        int tm, tn;
        proj_tile(t, p.tiles_m, p.tiles_n, tm, tn);
        const int slot = tm / p.tiles_per_slot;
        const int row0 = (tm - slot * p.tiles_per_slot) * kPairBM + 128 * static_cast<int>(rank);
        const int f0 = tn * kProjBN + 128 * static_cast<int>(rank);
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % kPairStages;
          // freed by rank 0's commit (for rank 1, a signal from the other SM)
          ok = mbar_wait(bar_empty + 8 * s, ((it / kPairStages) & 1) ^ 1u, abort_flag, kProjWaitNs);
          if (!ok) break;
          const uint32_t dst = sbase + s * kPairStageBytes;
          mbar_arrive_expect_tx(bar_full + 8 * s, kPairStageBytes);
          for (int bx = 0; bx < kPairBoxes; ++bx) {
            const int k0 = (kb * kPairBoxes + bx) * kProjBK;
            proj_load_a(&tmX, dst + bx * kPairBoxBytes, bar_full + 8 * s, p, k0, row0, slot, pol);
            tma_load_4d(dst + kPairHalfBytes + bx * kPairBoxBytes, &tmW, bar_full + 8 * s, k0, f0,
                        0, 0, pol);
          }
          issued = it + 1;
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // -------------------------------------------------------------- MMA issue
      constexpr uint32_t idesc = make_idesc_bf16(kPairBM, kProjBN, 0, 0);
      const uint64_t dA = make_sdesc_sw128(sbase, 16, 1024);
      const uint64_t dB = make_sdesc_sw128(sbase + kPairHalfBytes, 16, 1024);
      int it = 0, n = 0;
      for (int t = pair; t < ntiles && ok; t += npairs, ++n) {
        const int a = n & 1;                      // accumulator of this tile
        ok = mbar_wait(bar_acc_empty + 8 * a, ((n >> 1) & 1) ^ 1u, abort_flag, kProjWaitNs);
        if (!ok) break;
        tc_fence_after();
        const uint32_t acc = tmem + static_cast<uint32_t>(a * kProjBN);
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % kPairStages;
          ok = mbar_wait(bar_full + 8 * s, (it / kPairStages) & 1, abort_flag, kProjWaitNs);
          if (!ok) break;
          tc_fence_after();
          const uint32_t stage = static_cast<uint32_t>((s * kPairStageBytes) >> 4);
#pragma unroll
          for (int kk = 0; kk < kPairBoxes * kProjBK / 16; ++kk) {  // 32 bytes of K per MMA
            const uint32_t off = static_cast<uint32_t>(((kk >> 2) * kPairBoxBytes) >> 4) + (kk & 3) * 2;
            umma_ss_pair(acc, dA + stage + off, dB + stage + off, idesc,
                         (kb > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit_pair(bar_empty + 8 * s);
          umma_commit_pair(mapa_cluster(bar_empty + 8 * s, 1));
        }
        if (ok) {
          umma_commit_pair(bar_acc_full + 8 * a);
          umma_commit_pair(mapa_cluster(bar_acc_full + 8 * a, 1));
        }
      }
    } else if (lane == 0) {
      // ---------------------------------------- rank 1: forward load arrivals
      int it = 0;
      for (int t = pair; t < ntiles && ok; t += npairs)
        for (int kb = 0; kb < nk && ok; ++kb, ++it) {
          const int s = it % kPairStages;
          ok = mbar_wait(bar_full + 8 * s, (it / kPairStages) & 1, abort_flag, kProjWaitNs);
          if (ok) mbar_arrive_remote(mapa_cluster(bar_full + 8 * s, 0));
        }
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- epilogue
    const int wq = warp & 3;                 // TMEM lane quarter of this warp
    const int row = wq * 32 + lane;
    const uint32_t lanes = static_cast<uint32_t>(wq * 32) << 16;
    int n = 0;
    for (int t = pair; t < ntiles && ok; t += npairs, ++n) {
      const int a = n & 1;
      int tm, tn;
      proj_tile(t, p.tiles_m, p.tiles_n, tm, tn);
      const bool got = mbar_wait(bar_acc_full + 8 * a, (n >> 1) & 1, abort_flag, kProjWaitNs);
      if (!__all_sync(0xffffffffu, got)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int slot = tm / p.tiles_per_slot;
      const int ar0 = (tm - slot * p.tiles_per_slot) * kPairBM + 128 * static_cast<int>(rank);
      proj_store_block(p, tmem + lanes + static_cast<uint32_t>(a * kProjBN), slot, ar0,
                       tn * kProjBN, row, lane, [&] {
                         // the accumulator is in registers: hand it back to
                         // rank 0's MMA thread
                         tc_fence_before();
                         __syncwarp();
                         if (lane == 0) mbar_arrive_cluster(mapa_cluster(bar_acc_empty + 8 * a, 0));
                       });
    }
  }

  // ------------------------------------------------------------------ teardown
  if (!ok) {
    *abort_flag = 1;
    atomicExch(p.status, kProjStatusTimeout);
  }
  tc_fence_before();
  __syncthreads();
  if (*abort_flag) {
    // Let the asynchronous work this CTA issued land: its own last
    // kPairStages ring loads (they complete on its own barriers) and, on
    // rank 0, every MMA (one more commit, then its barrier).
    if (warp == 0 && lane == 0)
      for (int i = issued > kPairStages ? issued - kPairStages : 0; i < issued; ++i)
        mbar_wait_drain(bar_full + 8 * (i % kPairStages), (i / kPairStages) & 1, kProjWaitNs);
    if (warp == 1 && lane == 0 && rank == 0) {
      umma_commit_pair(bar_drain);
      mbar_wait_drain(bar_drain, 0, kProjWaitNs);
    }
    __syncthreads();
  }
  // No rank leaves while the other may still signal its barriers or use its
  // tensor memory.
  tc_fence_before();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kProjTmemCols);
  }
}

}  // namespace sp
