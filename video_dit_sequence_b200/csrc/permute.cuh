// permute.cuh -- the Ulysses token<->head exchange on one GPU.
//
// With P virtual ranks in one HBM, the all-to-all of "Splitting one
// generation across four GPUs" (fal.ai, "Generate video with WAN 2.2 across
// four GPUs") is a pure permutation of 16-bit words:
//   pack   : xh[j][b][r*Nl + n][hh][:] = xs[r][b][n][j*Hl + hh][:]
//   unpack : os[r][b][n][j*Hl + hh][:] = oh[j][b][r*Nl + n][hh][:]
// With one GPU per rank the same exchange is, on each rank, a reorder into P
// send chunks before the all-to-all and the reverse after the return one:
//   exchange pack   : send[j][b][n][hh][:]  = xs_r[b][n][j*Hl + hh][:]
//   exchange unpack : os_r[b][n][j*Hl + hh][:] = recv[j][b][n][hh][:]
// All four move contiguous runs of Hl*D words (>= 128 bytes), so every thread
// copies 16-byte vectors and consecutive threads touch consecutive vectors of
// one run on both sides.  The destination is walked linearly (vector v of
// the kernel writes bytes 16v .. 16v+15 of the output); the source address
// comes from the index arithmetic above, with invariant-divisor
// multiplications in place of integer division.
#pragma once
#include <cstdint>

namespace sp {

// Quotient / remainder by a fixed divisor d >= 1 for numerators n < 2^31:
// q = (mulhi(n, m) + n) >> s with s = ceil(log2 d) and
// m = floor(2^32 (2^s - d) / d) + 1 (Granlund & Montgomery, "Division by
// invariant integers using multiplication", PLDI 1994, section 4).
struct FastDiv {
  uint32_t d, m, s;
};

inline FastDiv make_fastdiv(uint32_t d) {
  FastDiv f;
  f.d = d;
  uint32_t s = 0;
  while ((1ull << s) < d) ++s;
  f.s = s;
  f.m = static_cast<uint32_t>((((1ull << s) - d) << 32) / d + 1ull);
  return f;
}

__device__ __forceinline__ uint32_t fdiv(uint32_t n, const FastDiv &f) {
  return (__umulhi(n, f.m) + n) >> f.s;
}

struct PermuteParams {
  const uint4 *src;
  uint4 *dst;
  uint32_t total_vec;      // output vectors (16 B each), < 2^31
  FastDiv vr;              // vectors per run: Hl*D/8
  FastDiv nl;              // Nl
  FastDiv p;               // P
  FastDiv bdiv;            // B
  FastDiv pvr;             // P * vectors per run (unpack: vectors per output row)
  FastDiv bnl;             // B * Nl (exchange modes)
  uint32_t H_vec;          // vectors per sequence-sharded token row: H*D/8
  uint32_t Hl_vec;         // vectors per head-sharded token row: Hl*D/8
  uint32_t Nl, Np, B, P;
  FastDiv hvec;            // H*D/8 (shard modes)
  FastDiv ntok;            // N (unshard)
  uint32_t N;
};

constexpr int kPermThreads = 256;
constexpr int kPermUnroll = 4;

// Loads bypass L1 (each byte is read once); stores stream.
__device__ __forceinline__ uint4 ld_stream(const uint4 *p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}
__device__ __forceinline__ void st_stream(uint4 *p, const uint4 &v) {
  asm volatile("st.global.cs.v4.u32 [%0], {%1,%2,%3,%4};"
               ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

// Source vector of pack for output vector v: output row R = v / Vr holds
// (j, b, r, n) with R = ((j*B + b)*P + r)*Nl + n; vector k = v % Vr of it.
__device__ __forceinline__ uint64_t pack_src(uint32_t v, const PermuteParams &p) {
  uint32_t R = fdiv(v, p.vr);
  uint32_t k = v - R * p.vr.d;
  uint32_t blk = fdiv(R, p.nl);
  uint32_t n = R - blk * p.Nl;
  uint32_t jb = fdiv(blk, p.p);
  uint32_t r = blk - jb * p.P;
  uint32_t j = fdiv(jb, p.bdiv);
  uint32_t b = jb - j * p.B;
  return (static_cast<uint64_t>(r * p.B + b) * p.Nl + n) * p.H_vec +
         static_cast<uint64_t>(j) * p.Hl_vec + k;
}

// Source vector of unpack for output vector v: output row R = v / (P*Vr)
// holds (r, b, n) with R = (r*B + b)*Nl + n; within it, run j = w / Vr and
// vector k = w % Vr, w = v % (P*Vr).
__device__ __forceinline__ uint64_t unpack_src(uint32_t v, const PermuteParams &p) {
  uint32_t R = fdiv(v, p.pvr);
  uint32_t w = v - R * p.pvr.d;
  uint32_t j = fdiv(w, p.vr);
  uint32_t k = w - j * p.vr.d;
  uint32_t rb = fdiv(R, p.nl);
  uint32_t n = R - rb * p.Nl;
  uint32_t r = fdiv(rb, p.bdiv);
  uint32_t b = rb - r * p.B;
  return (static_cast<uint64_t>(j * p.B + b) * p.Np + r * p.Nl + n) * p.Hl_vec + k;
}

// Exchange pack, output vector v: send row R = v / Vr = j*(B*Nl) + bn,
// vector k = v % Vr; the source row is bn of the rank's shard.
__device__ __forceinline__ uint64_t exchange_pack_src(uint32_t v, const PermuteParams &p) {
  uint32_t R = fdiv(v, p.vr);
  uint32_t k = v - R * p.vr.d;
  uint32_t j = fdiv(R, p.bnl);
  uint32_t bn = R - j * p.bnl.d;
  return static_cast<uint64_t>(bn) * p.H_vec + static_cast<uint64_t>(j) * p.Hl_vec + k;
}

// Exchange unpack, output vector v: shard row bn = v / (P*Vr); within it
// run j = w / Vr and vector k = w % Vr, w = v % (P*Vr).
__device__ __forceinline__ uint64_t exchange_unpack_src(uint32_t v, const PermuteParams &p) {
  uint32_t bn = fdiv(v, p.pvr);
  uint32_t w = v - bn * p.pvr.d;
  uint32_t j = fdiv(w, p.vr);
  uint32_t k = w - j * p.vr.d;
  return (static_cast<uint64_t>(j) * p.bnl.d + bn) * p.Hl_vec + k;
}

// Shard, output vector v: shard row R = v / (H*D/8) = (r*B + b)*Nl + n holds
// token t = r*Nl + n of batch b of the logical [B][N][H][D] tensor; a token
// slot at or past N is padding and reads as zero (kNoSource).
constexpr uint64_t kNoSource = ~0ull;
__device__ __forceinline__ uint64_t shard_src(uint32_t v, const PermuteParams &p) {
  uint32_t R = fdiv(v, p.hvec);
  uint32_t k = v - R * p.hvec.d;
  uint32_t rb = fdiv(R, p.nl);
  uint32_t n = R - rb * p.Nl;
  uint32_t r = fdiv(rb, p.bdiv);
  uint32_t b = rb - r * p.B;
  uint32_t t = r * p.Nl + n;
  if (t >= p.N) return kNoSource;
  return (static_cast<uint64_t>(b) * p.N + t) * p.hvec.d + k;
}

// Unshard, output vector v: logical row R = v / (H*D/8) = b*N + t; token t
// lives in shard t / Nl at local row t % Nl.
__device__ __forceinline__ uint64_t unshard_src(uint32_t v, const PermuteParams &p) {
  uint32_t R = fdiv(v, p.hvec);
  uint32_t k = v - R * p.hvec.d;
  uint32_t b = fdiv(R, p.ntok);
  uint32_t t = R - b * p.N;
  uint32_t r = fdiv(t, p.nl);
  uint32_t n = t - r * p.Nl;
  return (static_cast<uint64_t>(r * p.B + b) * p.Nl + n) * p.hvec.d + k;
}

enum PermuteMode {
  kModePack = 0, kModeUnpack = 1, kModeExchangePack = 2, kModeExchangeUnpack = 3,
  kModeShard = 4, kModeUnshard = 5
};

template <int kMode>
__device__ __forceinline__ uint64_t permute_src(uint32_t v, const PermuteParams &p) {
  if (kMode == kModePack) return pack_src(v, p);
  if (kMode == kModeUnpack) return unpack_src(v, p);
  if (kMode == kModeExchangePack) return exchange_pack_src(v, p);
  if (kMode == kModeShard) return shard_src(v, p);
  if (kMode == kModeUnshard) return unshard_src(v, p);
  return exchange_unpack_src(v, p);
}

template <int kMode>
__global__ void __launch_bounds__(kPermThreads)
permute_kernel(const PermuteParams p) {
  const uint32_t base = blockIdx.x * (kPermThreads * kPermUnroll) + threadIdx.x;
  uint4 v[kPermUnroll];
#pragma unroll
  for (int u = 0; u < kPermUnroll; ++u) {
    uint32_t o = base + u * kPermThreads;
    if (o < p.total_vec) {
      const uint64_t s = permute_src<kMode>(o, p);
      v[u] = (kMode == kModeShard && s == kNoSource) ? make_uint4(0u, 0u, 0u, 0u)
                                                     : ld_stream(p.src + s);
    }
  }
#pragma unroll
  for (int u = 0; u < kPermUnroll; ++u) {
    uint32_t o = base + u * kPermThreads;
    if (o < p.total_vec) st_stream(p.dst + o, v[u]);
  }
}

// ------------------------------------------------------------------ push
// One rank's K/V exchange over peer memory, for the multi-GPU form in which
// the attention kernel overlaps the arrival of the K/V chunks: rank `rank`
// stores its chunk for head group j straight into rank j's received-group
// buffers (the exchange pack fused with the transfer; no send buffer, no
// all-to-all), at chunk slot `rank`:
//   group_j[rank][b][n][hh][:] = x_rank[b][n][j*Hl + hh][:]     (x = K, V)
// and then counts itself done in rank j's arrival counter for source `rank`.
// A CTA covers kPermThreads * kPermUnroll vectors of one (tensor, j) chunk;
// rank j's counter for this rank reaches 2 * blocks_per_chunk per step (K
// and V), so after step e it is e * 2 * blocks_per_chunk.
constexpr int kMaxPushPeers = 8;

struct PushParams {
  const uint4 *src[2];                            // this rank's K and V shards
  uint4 *dst[2][kMaxPushPeers];                   // rank j's received K and V groups
  unsigned long long *count[kMaxPushPeers];       // rank j's arrival counters [P]
  FastDiv vr;                                     // vectors per run: Hl*D/8
  uint32_t chunk_vec;                             // vectors of one chunk: B*Nl*Hl*D/8
  uint32_t H_vec, Hl_vec;
  uint32_t rank;
};

__host__ __device__ constexpr uint32_t push_blocks_per_chunk(uint32_t chunk_vec) {
  return (chunk_vec + kPermThreads * kPermUnroll - 1) / (kPermThreads * kPermUnroll);
}

// Release-add at system scope: the stores this thread observed before it
// (the whole CTA's, through the barrier before the call) are visible to a
// thread of any GPU that acquires the counter value.
__device__ __forceinline__ void red_release_sys_add(unsigned long long *p, unsigned long long v) {
  asm volatile("red.release.sys.global.add.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

__global__ void __launch_bounds__(kPermThreads)
exchange_push_kernel(const __grid_constant__ PushParams p) {
  const int tensor = blockIdx.z, j = blockIdx.y;
  const uint4 *src = p.src[tensor];
  uint4 *dst = p.dst[tensor][j] + static_cast<uint64_t>(p.rank) * p.chunk_vec;
  const uint32_t base = blockIdx.x * (kPermThreads * kPermUnroll) + threadIdx.x;
  uint4 v[kPermUnroll];
#pragma unroll
  for (int u = 0; u < kPermUnroll; ++u) {
    const uint32_t o = base + u * kPermThreads;
    if (o < p.chunk_vec) {
      const uint32_t row = fdiv(o, p.vr);
      const uint32_t k = o - row * p.vr.d;
      v[u] = ld_stream(src + static_cast<uint64_t>(row) * p.H_vec +
                       static_cast<uint64_t>(j) * p.Hl_vec + k);
    }
  }
#pragma unroll
  for (int u = 0; u < kPermUnroll; ++u) {
    const uint32_t o = base + u * kPermThreads;
    if (o < p.chunk_vec) dst[o] = v[u];
  }
  __threadfence_system();
  __syncthreads();
  if (threadIdx.x == 0) red_release_sys_add(p.count[j] + p.rank, 1ull);
}

}  // namespace sp
