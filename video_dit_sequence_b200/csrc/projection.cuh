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
// tile of y is 256 x 512, each CTA of the pair holds 128 of its rows of A
// and, for each 256-feature half, 128 rows of w (64-wide K slices through a
// 4-stage ring of 48 KB stages), and one thread of the even CTA issues
// 256 x 256 x 16 tcgen05 MMAs (cta_group::2) that read both CTAs' shared
// memory and accumulate each CTA's 128 rows in that CTA's tensor memory.
// Against 256 x 256 tiles the SMs move a quarter less operand data from L2
// (x is read once per 512 features instead of per 256); against one CTA per
// 128 x 256 tile, half as much.  Each CTA's loads complete on its own
// barrier; the odd CTA forwards that completion to the even one with a
// remote mbarrier arrive (each CTA loads only its own operands; the plain
// arrive form, whose release is CTA-scoped: a cluster-scoped release per
// 512-cycle stage cost half the throughput).  Eight epilogue warps per CTA
// (two per TMEM lane quarter) add the bias, round to bf16 and write 32 x 32
// chunks through shared memory and TMA stores (where a tile's rows are
// consecutive destination rows; else 16-byte stores per row).  The two
// halves of a tile fill the tensor memory; the MMA thread staggers them at
// the ends of each tile so that one half drains while the other's MMAs run
// (see the kernel).  The kernel is persistent, one pair per two SMs; tiles
// run in groups of kProjGroupN column blocks so that the pairs working at
// one time share their w slice in L2.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "sm100.cuh"

namespace sp {

// 3-D tiled TMA store from this CTA's shared memory, tracked by the issuing
// thread's bulk groups (commit with bulk_commit, wait with bulk_wait_*).
// Elements of the box outside the tensor are not written.
__device__ __forceinline__ void tma_store_3d(const CUtensorMap *m, uint32_t src, int32_t c0,
                                             int32_t c1, int32_t c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];"
      ::"l"(reinterpret_cast<uint64_t>(m)), "r"(src), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// Waits until at most N of this thread's committed bulk groups still read
// their shared-memory source.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

// Waits until every committed bulk group of this thread has completed.
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

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
  // 1: the epilogue stores through TMA (the output maps), possible where a
  // tile's rows are consecutive rows of the destination; 0: 16-byte stores
  int32_t tma_store;
};

constexpr int kProjBN = 256;                      // features of a tile
constexpr int kProjBK = 64;                       // bf16 elements: one 128-byte row
constexpr int kProjGroupN = 6;
// Eight epilogue warps: two per TMEM lane quarter, each taking half of the
// 256 columns of an accumulator half (one warp per SM sub-partition would
// drain a half no faster than its dependent chain of loads, conversions and
// stores allows).
constexpr int kProjEpiWarps = 8;
constexpr int kProjThreads = 32 * (2 + kProjEpiWarps);   // TMA, MMA, epilogue warps
constexpr int kEpiChunks = kProjBN / 32 / (kProjEpiWarps / 4);  // 32-column chunks per warp
constexpr uint32_t kProjTmemCols = 512;           // a tile's two 256-column halves
constexpr uint64_t kProjWaitNs = 2000000000ull;   // 2 s per wait
constexpr int32_t kProjStatusTimeout = 7;         // SP_ERR_TIMEOUT

// A CTA pair per 256 x 512 tile: two 256-feature halves, each with its own
// 256-column accumulator in every CTA's TMEM.  A stage holds 64 elements of K
// in three 16 KB boxes per CTA: 128 rows of A and 128 rows of w for each half
// (the half's features 128r .. 128r + 127 on rank r), so that every stage's
// barrier round trip and commit cover eight MMAs.
constexpr int kPairBM = 256;
constexpr int kPairTileN = 2 * kProjBN;           // features of a tile
constexpr int kPairStages = 4;
constexpr int kPairBoxBytes = 128 * 128;          // 128 rows x 64 bf16: 16 KB
constexpr int kPairStageBytes = 3 * kPairBoxBytes;   // A, w of half 0, w of half 1
// Stages at each end of a tile whose MMAs of one half are deferred (see the
// MMA thread); at most kPairStages - 1 so that the ring still has a free slot.
constexpr int kPairDefer = kPairStages - 1;
// Epilogue staging for TMA stores: per epilogue warp two buffers of one
// 32-row x 32-feature chunk (64-byte rows, 64-byte swizzle).
constexpr int kStageChunkBytes = 32 * 64;
constexpr int kPairOffStage = kPairStages * kPairStageBytes;
constexpr int kPairOffBar = kPairOffStage + kProjEpiWarps * 2 * kStageChunkBytes;
constexpr int kPairOffMisc = kPairOffBar + (2 * kPairStages + 5) * 8;  // ..., bar_drain
constexpr int kPairSmemBytes = kPairOffMisc + 16 + 1024;
static_assert(kPairSmemBytes <= 227 * 1024, "projection shared memory");

// Tile t of the y matrix as (row block, column block): groups of
// kProjGroupN column blocks (3,072 features: 31 MB of a 5,120-wide w), the
// row blocks in order and a group's column blocks inside each.  The pairs at
// work at one time share the group's w, which stays in L2 while x streams
// through; grouping row blocks instead (w streaming, x resident) read a third
// more from DRAM with the 512-feature tiles.
__device__ __forceinline__ void proj_tile(int t, int tiles_m, int tiles_n, int &tm, int &tn) {
  const int per_group = kProjGroupN * tiles_m;
  const int g = t / per_group;
  const int first_n = g * kProjGroupN;
  const int gn = min(kProjGroupN, tiles_n - first_n);
  const int in_group = t - g * per_group;
  tn = first_n + in_group % gn;
  tm = in_group / gn;
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

// Stores this warp's share of an accumulator half: the 32 rows of its TMEM
// lane quarter (`row` = 32 * quarter + lane) and the 32 * kEpiChunks columns
// at taddr.  Row `row` of the half is A row ar0 + row of batch slot `slot`;
// the share's features are n0 .. n0 + 32 * kEpiChunks - 1.  `release()` runs
// once the share has been read (the accumulator is free when every epilogue
// warp of the pair has arrived), so that the MMAs may reuse it while the
// stores run.  Each lane stores its own row, 64 bytes per 32-feature chunk.
// The destination offset is a row part plus a feature part in every layout;
// the feature part's head and group indices are divided out once and then
// stepped chunk by chunk, and the next chunk's TMEM load is issued before
// this chunk is converted.
template <typename Release>
__device__ __forceinline__ void proj_store_block(const ProjParams &p, uint32_t taddr, int slot,
                                                 int ar0, int n0, int row, int lane,
                                                 Release release) {
  const int ar = ar0 + row;
  const int HD = p.H * p.D;
  // the row part of the destination offset, and whether the row exists
  int64_t rpart = 0;
  bool rok;
  if (p.out_proj) {
    // output projection: the y row of this token is its sequence-shard row
    rok = ar < p.rows_per_slot;
    int64_t yrow = ar;
    if (p.a_load == kALoadHeads) {  // token ar of batch slot `slot`
      const int r = ar / p.Nl, nn = ar - r * p.Nl;
      yrow = (static_cast<int64_t>(r) * p.B + slot) * p.Nl + nn;
    }
    rpart = yrow * p.nout;
  } else {
    // q, k, v projection (one batch slot: ar is the token row m of the
    // sequence-sharded hidden states)
    const int m = ar;
    rok = m < p.M;
    if (p.layout == kProjSeqSharded) {
      rpart = static_cast<int64_t>(m) * HD;
    } else if (p.layout == kProjHeadSharded) {
      const int bn = m % (p.B * p.Nl);                  // m = (r*B + b)*Nl + n
      const int r = m / (p.B * p.Nl), bb = bn / p.Nl, nn = bn - bb * p.Nl;
      rpart = (static_cast<int64_t>(bb) * p.Np + static_cast<int64_t>(r) * p.Nl + nn) *
              (p.Hl * p.D);
    } else {
      rpart = static_cast<int64_t>(m) * (p.Hl * p.D);
    }
  }
  // feature n0 as tensor tt, head h (group j, head hh in it), element d
  int tt = 0, h = 0, d = 0, j = 0, hh = 0;
  if (!p.out_proj) {
    tt = n0 / HD;
    const int hd = n0 - tt * HD;
    h = hd / p.D;
    d = hd - h * p.D;
    j = h / p.Hl;
    hh = h - j * p.Hl;
  }
  const int64_t group_rows = p.layout == kProjHeadSharded ? static_cast<int64_t>(p.B) * p.Np
                                                          : static_cast<int64_t>(p.M);
  // the three output tensors, read from the parameters with constant
  // indices: an array element picked by a run-time index is a slow load,
  // and every chunk's stores would wait for it
  __nv_bfloat16 *const out0 = p.out[0], *const out1 = p.out[1], *const out2 = p.out[2];
  uint32_t accv[2][32];
  __syncwarp();                                         // TMEM loads are warp-collective
  tmem_ld32(taddr, accv[0]);
#pragma unroll
  for (int ci = 0; ci < kEpiChunks; ++ci) {
    const int f = n0 + 32 * ci;                         // first feature of the chunk
    tmem_wait_ld();                                     // this chunk (and nothing later)
    if (ci + 1 < kEpiChunks) {
      __syncwarp();
      tmem_ld32(taddr + 32 * (ci + 1), accv[(ci + 1) & 1]);
    } else {
      release();
    }
    const uint32_t *acc = accv[ci & 1];
    if (f < p.nout && rok) {
      __nv_bfloat16 *base;
      int64_t fpart;
      if (p.out_proj) {
        base = p.y;
        fpart = f;
      } else {
        base = tt == 0 ? out0 : tt == 1 ? out1 : out2;
        fpart = p.layout == kProjSeqSharded
                    ? static_cast<int64_t>(h) * p.D + d
                    : (j * group_rows * p.Hl + hh) * p.D + d;
      }
      uint4 *dst = reinterpret_cast<uint4 *>(base + rpart + fpart);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        // nout is a multiple of 8: a vector lies wholly inside or past the row
        if (f + 8 * i < p.nout) {
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int col = 8 * i + 2 * e;
            float y0 = __uint_as_float(acc[col]), y1 = __uint_as_float(acc[col + 1]);
            if (p.bias != nullptr) {
              y0 += __bfloat162float(p.bias[f + col]);
              y1 += __bfloat162float(p.bias[f + col + 1]);
            }
            w[e] = pack_bf16x2(y0, y1);
          }
          dst[i] = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
    }
    // step the feature position by one chunk (D is a multiple of 32)
    d += 32;
    if (d == p.D) {
      d = 0;
      ++h;
      if (++hh == p.Hl) {
        hh = 0;
        ++j;
      }
      if (h == p.H) {
        h = 0;
        j = 0;
        hh = 0;
        ++tt;
      }
    }
  }
}

// The same share through TMA stores, for layouts whose tile rows are
// consecutive rows of the destination: map m0, m1 or m2 (q, k, v; y alone
// for the output projection) holds the destination as [Z][rows][W] (W
// features of a row, Z groups: the send layout's head groups, else 1).  Per
// 32-feature chunk the warp writes its 32 rows into one of two 2 KB staging
// buffers (64-byte rows, 64-byte swizzle, so that the 16-byte writes meet no
// bank conflict) and one lane stores the 32 x 32 box at column x, row y0,
// group z; rows and columns past the tensor are not written.  nbuf counts
// this warp's stores (it alternates the buffers across calls).
template <typename Release>
__device__ __forceinline__ void proj_store_block_tma(const ProjParams &p, const CUtensorMap *m0,
                                                     const CUtensorMap *m1, const CUtensorMap *m2,
                                                     uint32_t taddr, uint32_t stage, int y0,
                                                     int n0, int lane, int &nbuf,
                                                     Release release) {
  const int HD = p.H * p.D;
  const int groupw = p.Hl * p.D;                      // send layout: columns of a group
  // feature n0 as tensor tt, group z and column x of that tensor's map
  int tt = 0, z = 0, x = n0;
  if (!p.out_proj) {
    tt = n0 / HD;
    x = n0 - tt * HD;
    if (p.layout == kProjSendChunks) {
      z = x / groupw;
      x -= z * groupw;
    }
  }
  const uint32_t sw = static_cast<uint32_t>(lane >> 1) & 3u;   // this row's 64-byte swizzle
  uint32_t accv[2][32];
  __syncwarp();                                       // TMEM loads are warp-collective
  tmem_ld32(taddr, accv[0]);
#pragma unroll
  for (int ci = 0; ci < kEpiChunks; ++ci) {
    const int f = n0 + 32 * ci;                       // first feature of the chunk
    tmem_wait_ld();
    if (ci + 1 < kEpiChunks) {
      __syncwarp();
      tmem_ld32(taddr + 32 * (ci + 1), accv[(ci + 1) & 1]);
    } else {
      release();
    }
    if (f < p.nout) {
      const uint32_t *acc = accv[ci & 1];
      const uint32_t buf = stage + static_cast<uint32_t>(nbuf & 1) * kStageChunkBytes;
      // the store issued from this buffer two chunks ago has read it
      if (lane == 0) bulk_wait_read<1>();
      __syncwarp();
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int col = 8 * j + 2 * e;
          float v0 = __uint_as_float(acc[col]), v1 = __uint_as_float(acc[col + 1]);
          if (p.bias != nullptr && f + col < p.nout) {
            v0 += __bfloat162float(p.bias[f + col]);
            v1 += __bfloat162float(p.bias[f + col + 1]);
          }
          w[e] = pack_bf16x2(v0, v1);
        }
        st_shared_v4(buf + static_cast<uint32_t>(lane) * 64u + ((static_cast<uint32_t>(j) ^ sw) << 4),
                     make_uint4(w[0], w[1], w[2], w[3]));
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        tma_store_3d(tt == 0 ? m0 : tt == 1 ? m1 : m2, buf, x, y0, z);
        bulk_commit();
      }
      ++nbuf;
    }
    // the next chunk's column (D and the group width are multiples of 32)
    x += 32;
    if (!p.out_proj) {
      if (p.layout == kProjSendChunks) {
        if (x == groupw) {
          x = 0;
          if (++z == p.P) {
            z = 0;
            ++tt;
          }
        }
      } else if (x == HD) {
        x = 0;
        ++tt;
      }
    }
  }
}

// A CTA pair per 256 x 512 tile, launched as clusters of two CTAs.  Pair c
// (CTAs 2c and 2c + 1) computes tiles c, c + gridDim.x / 2, ...  CTA rank r
// holds A rows 128r .. 128r + 127 of each tile and, of each 256-feature half
// h, the w rows (features) 256h + 128r .. 256h + 128r + 127; its TMEM holds
// the tile's rows 128r .. 128r + 127, half h in columns 256h .. 256h + 255.
//   full[s]      rank 0: its own TMA bytes + one forwarded arrival from
//                rank 1 (rank 1's bytes landed); rank 1: its own TMA bytes
//   empty[s]     each rank: the MMA thread's commit after the stage's MMAs
//   acc_full[h]  each rank: the MMA thread's commit after a tile's last MMA
//                into half h
//   acc_empty[h] rank 0: one arrival per epilogue warp of both ranks once
//                half h is in registers
// The two halves fill all 512 TMEM columns, so a tile's MMAs cannot wait for
// a whole free accumulator as with two 256 x 256 tiles.  Instead the MMA
// thread staggers the halves at both ends of a tile: over its last
// kPairDefer stages it issues half 0 first and commits acc_full[0], so that
// the epilogue drains half 0 while half 1's last MMAs run; over the next
// tile's first kPairDefer stages it issues half 0 again (free by then) and
// holds those stages until half 1 has drained.  Each half still sums K in
// order.
__global__ void __launch_bounds__(kProjThreads, 1)
projection_pair_kernel(const __grid_constant__ CUtensorMap tmX,
                       const __grid_constant__ CUtensorMap tmW,
                       const __grid_constant__ CUtensorMap tmY0,
                       const __grid_constant__ CUtensorMap tmY1,
                       const __grid_constant__ CUtensorMap tmY2, const __grid_constant__ ProjParams p) {
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
  const int nk = (p.K + kProjBK - 1) / kProjBK;

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
      mbar_init(bar_acc_empty + 8 * a, 2 * kProjEpiWarps);  // epilogue warps of both ranks (rank 0 only)
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
        const int f0 = tn * kPairTileN + 128 * static_cast<int>(rank);
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const int s = it % kPairStages;
          // freed by rank 0's commit (for rank 1, a signal from the other SM)
          ok = mbar_wait(bar_empty + 8 * s, ((it / kPairStages) & 1) ^ 1u, abort_flag, kProjWaitNs);
          if (!ok) break;
          const uint32_t dst = sbase + s * kPairStageBytes;
          const uint32_t bar = bar_full + 8 * s;
          const int k0 = kb * kProjBK;
          mbar_arrive_expect_tx(bar, kPairStageBytes);
          proj_load_a(&tmX, dst, bar, p, k0, row0, slot, pol);
          tma_load_4d(dst + kPairBoxBytes, &tmW, bar, k0, f0, 0, 0, pol);
          tma_load_4d(dst + 2 * kPairBoxBytes, &tmW, bar, k0, f0 + kProjBN, 0, 0, pol);
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
      const uint64_t dB = make_sdesc_sw128(sbase + kPairBoxBytes, 16, 1024);
      int it = 0, n = 0;  // it: ring position of the tile's first stage
      // stage kb of the current tile has landed (both ranks' bytes)
      auto land = [&](int kb) {
        const int i = it + kb;
        const bool got = mbar_wait(bar_full + 8 * (i % kPairStages), (i / kPairStages) & 1,
                                   abort_flag, kProjWaitNs);
        tc_fence_after();
        return got;
      };
      // the four 256 x 256 x 16 MMAs of stage kb into half h
      auto mma = [&](int kb, int h) {
        const uint32_t stage =
            static_cast<uint32_t>((((it + kb) % kPairStages) * kPairStageBytes) >> 4);
        const uint64_t b = dB + stage + static_cast<uint32_t>((h * kPairBoxBytes) >> 4);
        const uint32_t acc = tmem + static_cast<uint32_t>(h * kProjBN);
#pragma unroll
        for (int kk = 0; kk < kProjBK / 16; ++kk)  // 32 bytes of K per MMA
          umma_ss_pair(acc, dA + stage + kk * 2, b + kk * 2, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
      };
      // stage kb may be refilled once the MMAs issued so far have read it
      auto release = [&](int kb) {
        const uint32_t bar = bar_empty + 8 * ((it + kb) % kPairStages);
        umma_commit_pair(bar);
        umma_commit_pair(mapa_cluster(bar, 1));
      };
      auto acc_done = [&](int h) {
        umma_commit_pair(bar_acc_full + 8 * h);
        umma_commit_pair(mapa_cluster(bar_acc_full + 8 * h, 1));
      };
      // half h of the previous tile is in the epilogue's registers
      auto acc_free = [&](int h) {
        const bool got = mbar_wait(bar_acc_empty + 8 * h, (n & 1) ^ 1u, abort_flag, kProjWaitNs);
        tc_fence_after();
        return got;
      };
      for (int t = pair; t < ntiles && ok; t += npairs, ++n) {
        // stages [0, a): half 0, then (once half 1 is free) half 1;
        // [a, c): both halves per stage; [c, nk): half 0, acc_full[0], half 1
        const int a = min(kPairDefer, nk), c = max(a, nk - kPairDefer);
        ok = acc_free(0);
        for (int kb = 0; kb < a && ok; ++kb)
          if ((ok = land(kb))) mma(kb, 0);
        if (ok && a == nk) acc_done(0);
        if (ok) ok = acc_free(1);
        for (int kb = 0; kb < a && ok; ++kb) {
          mma(kb, 1);
          release(kb);
        }
        for (int kb = a; kb < c && ok; ++kb)
          if ((ok = land(kb))) {
            mma(kb, 0);
            mma(kb, 1);
            release(kb);
          }
        if (a < nk) {
          for (int kb = c; kb < nk && ok; ++kb)
            if ((ok = land(kb))) mma(kb, 0);
          if (ok) acc_done(0);
          for (int kb = c; kb < nk && ok; ++kb) {
            mma(kb, 1);
            release(kb);
          }
        }
        if (ok) acc_done(1);
        it += nk;
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
    // first column of this warp's share of each accumulator half
    const int col0 = ((warp - 2) >> 2) * (kEpiChunks * 32);
    int n = 0, nbuf = 0;
    const uint32_t stage = sbase + kPairOffStage + static_cast<uint32_t>((warp - 2) * 2 * kStageChunkBytes);
    for (int t = pair; t < ntiles && ok; t += npairs, ++n) {
      int tm, tn;
      proj_tile(t, p.tiles_m, p.tiles_n, tm, tn);
      const int slot = tm / p.tiles_per_slot;
      const int ar0 = (tm - slot * p.tiles_per_slot) * kPairBM + 128 * static_cast<int>(rank);
      for (int h = 0; h < 2; ++h) {
        const bool got = mbar_wait(bar_acc_full + 8 * h, n & 1, abort_flag, kProjWaitNs);
        if (!__all_sync(0xffffffffu, got)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // the half is in registers (tcgen05.wait::ld has returned): hand it
        // back to rank 0's MMA thread.  The plain arrive releases at CTA
        // scope only: a cluster-scope release would first wait for every
        // global store this thread has issued, which the MMAs do not need.
        auto release = [&] {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_remote(mapa_cluster(bar_acc_empty + 8 * h, 0));
        };
        const uint32_t taddr = tmem + lanes + static_cast<uint32_t>(h * kProjBN + col0);
        const int n0 = tn * kPairTileN + h * kProjBN + col0;
        if (p.tma_store)
          proj_store_block_tma(p, &tmY0, &tmY1, &tmY2, taddr, stage, ar0 + wq * 32, n0, lane,
                               nbuf, release);
        else
          proj_store_block(p, taddr, slot, ar0, n0, row, lane, release);
      }
    }
    // the staging buffers stay allocated until the last store has read them
    if (lane == 0) bulk_wait_all();
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
