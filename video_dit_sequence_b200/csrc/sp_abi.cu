// sp_abi.cu -- the C ABI declared in include/sp.h: argument checks, TMA
// descriptor construction and kernel launches.  One translation unit holds
// every kernel so that the device status word needs no relocatable code.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include <nvtx3/nvToolsExt.h>

#include "attention.cuh"
#include "permute.cuh"
#include "projection.cuh"
#include "sp.h"

namespace {

// One NVTX range per ABI call that enqueues work, so that a profiler's
// timeline shows the C-ABI entry points; with no profiler attached a
// push/pop pair is a few nanoseconds.
struct NvtxRange {
  explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange &) = delete;
  NvtxRange &operator=(const NvtxRange &) = delete;
};

__device__ int32_t g_status = 0;
// Where status_take_kernel leaves the value it took out of g_status.
__device__ int32_t g_status_taken = 0;

// Takes the status word and clears it in one atomic exchange on the device,
// so that a timeout recorded by a kernel on another stream is either taken
// here or left for the next call, never lost between a read and a clear.
__global__ void status_take_kernel() { g_status_taken = atomicExch(&g_status, 0); }

std::atomic<uint64_t> g_launches{0};

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// heads_split: the call splits heads into P groups, so P must divide H.
sp_status check_common(const sp_shape *s, bool heads_split = true) {
  if (s == nullptr) return SP_ERR_NULL;
  if (s->B < 1 || s->N < 1 || s->H < 1 || s->P < 1 || s->D < 1) return SP_ERR_SHAPE;
  if (heads_split && s->H % s->P != 0) return SP_ERR_HEADS_NOT_DIVISIBLE;
  if (s->D != 64 && s->D != 128) return SP_ERR_UNSUPPORTED_D;
  if (s->P > 65535 || s->B > 65535 || s->H > 65535) return SP_ERR_SHAPE;
  const int64_t Nl = (static_cast<int64_t>(s->N) + s->P - 1) / s->P;
  const int64_t elems = static_cast<int64_t>(s->P) * s->B * Nl * s->H * s->D;
  // permute kernels index 16-byte vectors with 32-bit integers below 2^31
  if (elems / 8 >= (int64_t(1) << 31)) return SP_ERR_SHAPE;
  return SP_OK;
}

sp_status launch_status(cudaError_t e) {
  if (e != cudaSuccess) return SP_ERR_CUDA;
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return SP_OK;
}

constexpr int kMaxDevices = 64;
std::mutex g_mu;

// Device address of g_status on the current device (looked up once per
// device; host code must not use the symbol itself as a pointer).
int32_t *status_ptr() {
  static int32_t *ptrs[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> g(g_mu);
  if (ptrs[dev] == nullptr) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status) == cudaSuccess) ptrs[dev] = static_cast<int32_t *>(p);
  }
  return ptrs[dev];
}

sp_status permute(const void *src, void *dst, const sp_shape *s, void *stream, int mode) {
  // sharding splits tokens only: any P
  const bool shard = mode == sp::kModeShard || mode == sp::kModeUnshard;
  sp_status st = check_common(s, !shard);
  if (st != SP_OK) return st;
  if (src == nullptr || dst == nullptr) return SP_ERR_NULL;
  if (!aligned16(src) || !aligned16(dst)) return SP_ERR_ALIGN;
  const uint32_t P = s->P, B = s->B, H = s->H, D = s->D;
  const uint32_t Hl = shard ? H : H / P;  // (unused by the shard modes)
  const uint32_t Nl = (s->N + P - 1) / P;
  sp::PermuteParams p;
  std::memset(&p, 0, sizeof(p));
  p.src = static_cast<const uint4 *>(src);
  p.dst = static_cast<uint4 *>(dst);
  const bool exchange = mode == sp::kModeExchangePack || mode == sp::kModeExchangeUnpack;
  // one rank's shard (exchange modes), all P shards, or the logical tensor
  p.total_vec = static_cast<uint32_t>(
      mode == sp::kModeUnshard ? static_cast<uint64_t>(B) * s->N * H * D / 8
                               : static_cast<uint64_t>(exchange ? 1 : P) * B * Nl * H * D / 8);
  p.hvec = sp::make_fastdiv(H * D / 8);
  p.ntok = sp::make_fastdiv(static_cast<uint32_t>(s->N));
  p.N = static_cast<uint32_t>(s->N);
  p.vr = sp::make_fastdiv(Hl * D / 8);
  p.nl = sp::make_fastdiv(Nl);
  p.p = sp::make_fastdiv(P);
  p.bdiv = sp::make_fastdiv(B);
  p.pvr = sp::make_fastdiv(P * Hl * D / 8);
  p.bnl = sp::make_fastdiv(B * Nl);
  p.H_vec = H * D / 8;
  p.Hl_vec = Hl * D / 8;
  p.Nl = Nl;
  p.Np = Nl * P;
  p.B = B;
  p.P = P;
  const uint32_t per_block = sp::kPermThreads * sp::kPermUnroll;
  const uint32_t blocks = (p.total_vec + per_block - 1) / per_block;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  switch (mode) {
    case sp::kModePack: sp::permute_kernel<sp::kModePack><<<blocks, sp::kPermThreads, 0, cs>>>(p); break;
    case sp::kModeUnpack: sp::permute_kernel<sp::kModeUnpack><<<blocks, sp::kPermThreads, 0, cs>>>(p); break;
    case sp::kModeExchangePack:
      sp::permute_kernel<sp::kModeExchangePack><<<blocks, sp::kPermThreads, 0, cs>>>(p);
      break;
    case sp::kModeShard: sp::permute_kernel<sp::kModeShard><<<blocks, sp::kPermThreads, 0, cs>>>(p); break;
    case sp::kModeUnshard:
      sp::permute_kernel<sp::kModeUnshard><<<blocks, sp::kPermThreads, 0, cs>>>(p);
      break;
    default:
      sp::permute_kernel<sp::kModeExchangeUnpack><<<blocks, sp::kPermThreads, 0, cs>>>(p);
      break;
  }
  return launch_status(cudaGetLastError());
}

// Tensor map over one of Q/K/V, viewed as [Bx][N rows][Hx heads][D] with
// the given row and batch strides (elements).  Rows >= N read as zero.
// es: element size in bytes (2: bf16, 1: E4M3 moved as bytes).  The box is
// 128 bytes wide: 64 bf16 or 128 E4M3 elements.
bool make_map(CUtensorMap *m, const void *base, int D, int Hx, int N, int Bx, int64_t row_el,
              int64_t batch_el, int es = 2, int box_rows = 128) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return false;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(Hx),
                        static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(Bx)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(D) * es, static_cast<cuuint64_t>(row_el) * es,
                           static_cast<cuuint64_t>(batch_el) * es};
  cuuint32_t box[4] = {static_cast<cuuint32_t>(128 / es), 1, static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(m, es == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 4,
                   const_cast<void *>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Tensor map over rank-major sequence shards [P][B][Nl][H][D] (B > 1 and
// P > 1), dims inner to outer (D, H, Nl, B, P).  Used only for token tiles
// that lie inside one shard; the box is box_rows rows (or Nl when smaller,
// in which case no tile uses the map).
bool make_map5(CUtensorMap *m, const void *base, int D, int H, int Nl, int B, int P,
               int es = 2, int box_rows = 128) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return false;
  const cuuint64_t row = static_cast<cuuint64_t>(H) * D * es;
  cuuint64_t dims[5] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(H),
                        static_cast<cuuint64_t>(Nl), static_cast<cuuint64_t>(B),
                        static_cast<cuuint64_t>(P)};
  cuuint64_t strides[4] = {static_cast<cuuint64_t>(D) * es, row, row * Nl,
                           row * Nl * static_cast<cuuint64_t>(B)};
  cuuint32_t box[5] = {static_cast<cuuint32_t>(128 / es), 1,
                       static_cast<cuuint32_t>(Nl < box_rows ? Nl : box_rows), 1, 1};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = enc(m, es == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 5,
                   const_cast<void *>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Tensor map over one rank's sequence shard [B][Nl][H][D] bf16, dims inner
// to outer (D, H, Nl, B): the Q source of the peer step.
bool make_map_shard(CUtensorMap *m, const void *base, int D, int H, int Nl, int B) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return false;
  const cuuint64_t row = static_cast<cuuint64_t>(H) * D * 2;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(H),
                        static_cast<cuuint64_t>(Nl), static_cast<cuuint64_t>(B)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(D) * 2, row, row * Nl};
  cuuint32_t box[4] = {64, 1, static_cast<cuuint32_t>(Nl < 128 ? Nl : 128), 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int D, bool kF8 = false>
cudaError_t launch_attention(const CUtensorMap &q, const CUtensorMap &k, const CUtensorMap &v,
                             const sp::AttnParams &p, int B, cudaStream_t cs) {
  using C = sp::AttnCfg<D, kF8>;
  static bool attr_set[kMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  {
    std::lock_guard<std::mutex> g(g_mu);
    if (!attr_set[dev]) {
      e = cudaFuncSetAttribute(sp::attention_kernel<D, kF8>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
      if (e != cudaSuccess) return e;
      attr_set[dev] = true;
    }
  }
  // every output row up to Np, padding rows included, belongs to some CTA
  dim3 grid((p.Np + 2 * C::kBM - 1) / (2 * C::kBM), p.H, B);
  sp::attention_kernel<D, kF8><<<grid, C::kThreads, C::kSmemBytes, cs>>>(q, k, v, p);
  return cudaGetLastError();
}

// Sets the kernel's dynamic shared-memory limit once per device.
template <typename Kernel>
cudaError_t set_smem_once(Kernel kernel, int bytes, bool (&done)[kMaxDevices]) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> g(g_mu);
  if (!done[dev]) {
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    done[dev] = true;
  }
  return cudaSuccess;
}

// Shared launch path.  The head-sharded and the sequence-sharded layouts are
// both [slots][rows][heads-per-slot][D] with different strides; the kernel
// finds (slot, head-in-slot) of global head h as (h / hsplit * B + b,
// h % hsplit).
sp_status attention(const void *q, const void *k, const void *v, void *o, float *lse,
                    const sp_shape *s, void *stream, bool seqsharded,
                    const float *dq = nullptr, const float *dk = nullptr,
                    const float *dv = nullptr, const uint32_t *mask = nullptr) {
  const bool f8 = dq != nullptr;
  if (f8 && (dk == nullptr || dv == nullptr)) return SP_ERR_NULL;
  const int es = f8 ? 1 : 2;
  // The fused call shards tokens only; heads are never split, so it takes
  // any P (the per-rank call of the multi-GPU form has Hl heads and P shards).
  sp_status st = check_common(s, !seqsharded);
  if (st != SP_OK) return st;
  if (q == nullptr || k == nullptr || v == nullptr || o == nullptr) return SP_ERR_NULL;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) ||
      (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u) != 0) ||
      (f8 && ((reinterpret_cast<uintptr_t>(dq) | reinterpret_cast<uintptr_t>(dk) |
               reinterpret_cast<uintptr_t>(dv)) & 3u) != 0))
    return SP_ERR_ALIGN;
  if ((f8 || mask != nullptr) && s->D != 128) return SP_ERR_UNSUPPORTED_D;
  if (mask != nullptr) {
    if ((reinterpret_cast<uintptr_t>(mask) & 3u) != 0) return SP_ERR_ALIGN;
    static_assert(sp::AttnCfg<128>::kMaxPlanCubes == SP_SPARSE_MAX_CUBES, "plan capacity");
    if ((s->N + SP_SPARSE_CUBE - 1) / SP_SPARSE_CUBE > SP_SPARSE_MAX_CUBES) return SP_ERR_SHAPE;
  }
  const int P = s->P, B = s->B, H = s->H, D = s->D, N = s->N;
  const int Hl = H / P;
  const int Nl = (N + P - 1) / P;
  const int Np = Nl * P;
  int Hx, Bx, hsplit;
  int64_t row_el, batch_el;
  const bool rank_major = seqsharded && B > 1 && P > 1;
  if (seqsharded) {
    Hx = H;
    hsplit = H;
    Bx = B;
    row_el = static_cast<int64_t>(H) * D;
    batch_el = static_cast<int64_t>(Nl) * H * D;  // one rank's [B][Nl] rows
  } else {
    Hx = Hl;
    hsplit = Hl;
    Bx = P * B;
    row_el = static_cast<int64_t>(Hl) * D;
    batch_el = static_cast<int64_t>(Np) * Hl * D;
  }
  int32_t *status = status_ptr();
  if (status == nullptr) return SP_ERR_CUDA;
  CUtensorMap mq, mk, mv;
  // the block-sparse kernel loads K and V one 64-token cube at a time
  const int kv_rows = mask != nullptr ? 64 : 128;
  if (rank_major) {
    if (!make_map5(&mq, q, D, H, Nl, B, P, es) ||
        !make_map5(&mk, k, D, H, Nl, B, P, es, kv_rows) ||
        !make_map5(&mv, v, D, H, Nl, B, P, es, kv_rows))
      return SP_ERR_CUDA;
  } else if (!make_map(&mq, q, D, Hx, N, Bx, row_el, batch_el, es) ||
             !make_map(&mk, k, D, Hx, N, Bx, row_el, batch_el, es, kv_rows) ||
             !make_map(&mv, v, D, Hx, N, Bx, row_el, batch_el, es, kv_rows)) {
    return SP_ERR_CUDA;
  }
  sp::AttnParams p;
  std::memset(&p, 0, sizeof(p));
  p.N = N;
  p.Np = Np;
  p.H = H;
  p.B = B;
  p.hsplit = hsplit;
  p.num_kv_tiles = (N + 127) / 128;
  const float scale = s->scale > 0.f ? s->scale : 1.0f / std::sqrt(static_cast<float>(D));
  p.scale_log2e = scale * 1.4426950408889634f;
  p.o = static_cast<__nv_bfloat16 *>(o);
  p.o_row = row_el;
  p.o_batch = batch_el;
  p.lse = lse;
  p.status = status;
  p.nl_split = rank_major ? Nl : 0;
  p.o_rank = static_cast<int64_t>(B) * Nl * H * D;
  p.q = static_cast<const uint8_t *>(q);
  p.k = static_cast<const uint8_t *>(k);
  p.v = static_cast<const uint8_t *>(v);
  p.dq = dq;
  p.dk = dk;
  p.dv = dv;
  p.nblk = p.num_kv_tiles;
  p.mask = mask;
  p.ncube = (N + 63) / 64;
  p.nwords = (p.ncube + 31) / 32;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  if (mask != nullptr) {
    using C = sp::AttnCfg<128>;
    static bool attr_set[kMaxDevices] = {};
    cudaError_t e = set_smem_once(sp::attention_sparse_kernel, C::kSmemBytesSparse, attr_set);
    if (e != cudaSuccess) return SP_ERR_CUDA;
    dim3 grid((Np + 2 * C::kBM - 1) / (2 * C::kBM), H, B);
    // 12 warps: the block-sparse kernel splits registers between warpgroups
    sp::attention_sparse_kernel<<<grid, 384, C::kSmemBytesSparse, cs>>>(mq, mk, mv, p);
    return launch_status(cudaGetLastError());
  }
  cudaError_t e = f8        ? launch_attention<128, true>(mq, mk, mv, p, B, cs)
                  : D == 64 ? launch_attention<64>(mq, mk, mv, p, B, cs)
                            : launch_attention<128>(mq, mk, mv, p, B, cs);
  return launch_status(e);
}

// One rank's step of the multi-GPU form with the Q and O exchanges fused
// into the attention kernel (see sp_attention_ulysses_peer in sp.h).
sp_status attention_peer(const void *const *q_shards, const void *k_group, const void *v_group,
                         void *const *o_shards, float *lse, int32_t rank, const sp_shape *s,
                         void *stream, const uint64_t *counts = nullptr, uint64_t epoch = 0,
                         uint64_t wait_ns = 0) {
  sp_status st = check_common(s, true);
  if (st != SP_OK) return st;
  if (s->D != 128) return SP_ERR_UNSUPPORTED_D;
  if (s->P > sp::kMaxPeers || rank < 0 || rank >= s->P) return SP_ERR_SHAPE;
  if (q_shards == nullptr || o_shards == nullptr || k_group == nullptr || v_group == nullptr)
    return SP_ERR_NULL;
  const int P = s->P, B = s->B, H = s->H, D = s->D, N = s->N;
  for (int r = 0; r < P; ++r) {
    if (q_shards[r] == nullptr || o_shards[r] == nullptr) return SP_ERR_NULL;
    if (!aligned16(q_shards[r]) || !aligned16(o_shards[r])) return SP_ERR_ALIGN;
  }
  if (!aligned16(k_group) || !aligned16(v_group) ||
      (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u) != 0))
    return SP_ERR_ALIGN;
  const int Hl = H / P;
  const int Nl = (N + P - 1) / P;
  const int Np = Nl * P;
  int32_t *status = status_ptr();
  if (status == nullptr) return SP_ERR_CUDA;
  sp::PeerArgs pa;
  std::memset(&pa, 0, sizeof(pa));
  for (int r = 0; r < P; ++r) {
    if (!make_map_shard(&pa.q[r], q_shards[r], D, H, Nl, B)) return SP_ERR_CUDA;
    pa.q_ptr[r] = static_cast<const uint8_t *>(q_shards[r]);
    pa.o_ptr[r] = static_cast<__nv_bfloat16 *>(o_shards[r]);
  }
  pa.nranks = P;
  pa.nl = Nl;
  pa.heads = H;
  pa.head0 = rank * Hl;
  // K and V: this rank's received head group [P][B][Nl][Hl][D], addressed
  // as the fused call addresses a sequence-sharded tensor with Hl heads.
  const bool rank_major = B > 1 && P > 1;
  CUtensorMap mk, mv;
  if (rank_major) {
    if (!make_map5(&mk, k_group, D, Hl, Nl, B, P) || !make_map5(&mv, v_group, D, Hl, Nl, B, P))
      return SP_ERR_CUDA;
  } else {
    const int64_t row_el = static_cast<int64_t>(Hl) * D;
    const int64_t batch_el = static_cast<int64_t>(Nl) * Hl * D;
    if (!make_map(&mk, k_group, D, Hl, N, B, row_el, batch_el) ||
        !make_map(&mv, v_group, D, Hl, N, B, row_el, batch_el))
      return SP_ERR_CUDA;
  }
  sp::AttnParams p;
  std::memset(&p, 0, sizeof(p));
  p.N = N;
  p.Np = Np;
  p.H = Hl;
  p.B = B;
  p.hsplit = Hl;
  p.num_kv_tiles = (N + 127) / 128;
  const float scale = s->scale > 0.f ? s->scale : 1.0f / std::sqrt(static_cast<float>(D));
  p.scale_log2e = scale * 1.4426950408889634f;
  p.lse = lse;
  p.status = status;
  p.nl_split = rank_major ? Nl : 0;
  p.k = static_cast<const uint8_t *>(k_group);
  p.v = static_cast<const uint8_t *>(v_group);
  p.nblk = p.num_kv_tiles;
  if (counts != nullptr) {
    // every source rank's chunk is counted by its push kernel's CTAs (K and V)
    const uint32_t chunk_vec = static_cast<uint32_t>(static_cast<int64_t>(B) * Nl * Hl * D / 8);
    p.counts = reinterpret_cast<const unsigned long long *>(counts);
    p.count_target = epoch * 2ull * sp::push_blocks_per_chunk(chunk_vec);
    p.count_nl = Nl;
    p.count_wait_ns = wait_ns > 0 ? wait_ns : sp::kWaitLimitNs;
  }
  using C = sp::AttnCfg<128>;
  static bool attr_set[kMaxDevices] = {};
  cudaError_t e = set_smem_once(sp::attention_peer_kernel, C::kSmemBytes, attr_set);
  if (e != cudaSuccess) return SP_ERR_CUDA;
  dim3 grid((Np + 2 * C::kBM - 1) / (2 * C::kBM), Hl, B);
  sp::attention_peer_kernel<<<grid, C::kThreads, C::kSmemBytes,
                              static_cast<cudaStream_t>(stream)>>>(pa, mk, mv, p);
  return launch_status(cudaGetLastError());
}

// One rank's K/V exchange over peer memory (see sp_exchange_push in sp.h).
sp_status exchange_push(const void *k_r, const void *v_r, void *const *k_groups,
                        void *const *v_groups, uint64_t *const *counts, uint64_t epoch,
                        int32_t rank, const sp_shape *s, void *stream) {
  sp_status st = check_common(s, true);
  if (st != SP_OK) return st;
  if (s->P > sp::kMaxPushPeers || rank < 0 || rank >= s->P) return SP_ERR_SHAPE;
  if (epoch < 1) return SP_ERR_SHAPE;
  if (k_r == nullptr || v_r == nullptr || k_groups == nullptr || v_groups == nullptr ||
      counts == nullptr)
    return SP_ERR_NULL;
  if (!aligned16(k_r) || !aligned16(v_r)) return SP_ERR_ALIGN;
  const int P = s->P, B = s->B, H = s->H, D = s->D;
  const int Hl = H / P;
  const int Nl = (s->N + P - 1) / P;
  sp::PushParams p;
  std::memset(&p, 0, sizeof(p));
  p.src[0] = static_cast<const uint4 *>(k_r);
  p.src[1] = static_cast<const uint4 *>(v_r);
  for (int j = 0; j < P; ++j) {
    if (k_groups[j] == nullptr || v_groups[j] == nullptr || counts[j] == nullptr)
      return SP_ERR_NULL;
    if (!aligned16(k_groups[j]) || !aligned16(v_groups[j]) ||
        (reinterpret_cast<uintptr_t>(counts[j]) & 7u) != 0)
      return SP_ERR_ALIGN;
    p.dst[0][j] = static_cast<uint4 *>(k_groups[j]);
    p.dst[1][j] = static_cast<uint4 *>(v_groups[j]);
    p.count[j] = reinterpret_cast<unsigned long long *>(counts[j]);
  }
  p.chunk_vec = static_cast<uint32_t>(static_cast<int64_t>(B) * Nl * Hl * D / 8);
  p.vr = sp::make_fastdiv(Hl * D / 8);
  p.H_vec = H * D / 8;
  p.Hl_vec = Hl * D / 8;
  p.rank = static_cast<uint32_t>(rank);
  dim3 grid(sp::push_blocks_per_chunk(p.chunk_vec), P, 2);
  sp::exchange_push_kernel<<<grid, sp::kPermThreads, 0, static_cast<cudaStream_t>(stream)>>>(p);
  return launch_status(cudaGetLastError());
}

// Tensor map over a row-major bf16 matrix [rows][cols] (cols contiguous), as
// 4-D with unit outer dims; boxes of 64 columns x box_rows rows under the
// 128-byte swizzle.  Rows past the end read as zeros.
bool make_map_matrix(CUtensorMap *m, const void *base, int cols, int rows, int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return false;
  const cuuint64_t row = static_cast<cuuint64_t>(cols) * 2;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows), 1, 1};
  cuuint64_t strides[3] = {row, row * rows, row * rows};
  cuuint32_t box[4] = {64, static_cast<cuuint32_t>(box_rows), 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

sp_status launch_projection(const CUtensorMap &ma, const void *w, int slots, sp::ProjParams p,
                            void *stream);

// Destination map of the projection epilogue's TMA stores: [Z][rows][W] bf16
// (W features a row), boxes of 32 rows x 32 features whose 64-byte rows the
// 64-byte swizzle spreads over the shared-memory banks.
bool make_map_out(CUtensorMap *m, void *base, int64_t W, int64_t rows, int64_t Z) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return false;
  const cuuint64_t row = static_cast<cuuint64_t>(W) * 2;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(W), static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(Z)};
  cuuint64_t strides[2] = {row, row * static_cast<cuuint64_t>(rows)};
  cuuint32_t box[3] = {32, 32, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                   CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

sp_status qkv_projection(const void *x, const void *w, const void *bias, void *q, void *k,
                         void *v, int32_t hidden, int32_t layout, const sp_shape *s,
                         void *stream) {
  if (layout < SP_QKV_SEQ_SHARDED || layout > SP_QKV_SEND_CHUNKS) return SP_ERR_SHAPE;
  sp_status st = check_common(s, layout != SP_QKV_SEQ_SHARDED);
  if (st != SP_OK) return st;
  if (x == nullptr || w == nullptr || q == nullptr || k == nullptr || v == nullptr)
    return SP_ERR_NULL;
  if (hidden < 8 || hidden % 8 != 0) return SP_ERR_SHAPE;
  if (!aligned16(x) || !aligned16(w) || !aligned16(q) || !aligned16(k) || !aligned16(v) ||
      (bias != nullptr && (reinterpret_cast<uintptr_t>(bias) & 1u) != 0))
    return SP_ERR_ALIGN;
  const int P = s->P, B = s->B, H = s->H, D = s->D, N = s->N;
  const int Nl = (N + P - 1) / P;
  const int64_t M64 = static_cast<int64_t>(layout == SP_QKV_SEND_CHUNKS ? 1 : P) * B * Nl;
  const int64_t nout64 = 3ll * H * D;
  if (M64 >= (int64_t(1) << 31) || nout64 >= (int64_t(1) << 31) ||
      M64 * hidden >= (int64_t(1) << 40))
    return SP_ERR_SHAPE;
  int32_t *status = status_ptr();
  if (status == nullptr) return SP_ERR_CUDA;
  CUtensorMap mx;
  if (!make_map_matrix(&mx, x, hidden, static_cast<int>(M64), 128)) return SP_ERR_CUDA;
  sp::ProjParams p;
  std::memset(&p, 0, sizeof(p));
  p.M = static_cast<int32_t>(M64);
  p.K = hidden;
  p.nout = static_cast<int32_t>(nout64);
  p.H = H;
  p.D = D;
  p.Hl = layout == SP_QKV_SEQ_SHARDED ? H : H / P;
  p.P = P;
  p.B = B;
  p.Nl = Nl;
  p.Np = Nl * P;
  p.layout = layout;
  p.out[0] = static_cast<__nv_bfloat16 *>(q);
  p.out[1] = static_cast<__nv_bfloat16 *>(k);
  p.out[2] = static_cast<__nv_bfloat16 *>(v);
  p.bias = static_cast<const __nv_bfloat16 *>(bias);
  p.status = status;
  p.a_load = sp::kALoadMatrix;
  p.rows_per_slot = p.M;
  // a tile's rows are consecutive destination rows except in the head-sharded
  // layout, whose rows jump between token shards and batch entries
  p.tma_store = layout != SP_QKV_HEAD_SHARDED;
  return launch_projection(mx, w, 1, p, stream);
}

// Tensor map over a bf16 operand viewed as 4-D [d3][d2][d1 rows][d0 cols]
// (cols contiguous; strides in elements), boxes of 64 columns x box_rows rows
// under the 128-byte swizzle.  Coordinates past an extent read as zeros.
bool make_map_rows4(CUtensorMap *m, const void *base, int64_t d0, int64_t d1, int64_t d2,
                    int64_t d3, int64_t s1, int64_t s2, int64_t s3, int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (enc == nullptr) return false;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(d0), static_cast<cuuint64_t>(d1),
                        static_cast<cuuint64_t>(d2), static_cast<cuuint64_t>(d3)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(s1) * 2, static_cast<cuuint64_t>(s2) * 2,
                           static_cast<cuuint64_t>(s3) * 2};
  cuuint32_t box[4] = {64, static_cast<cuuint32_t>(box_rows), 1, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims,
                   strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// The projection after attention (see sp_out_projection in sp.h): the GEMM
// of the q, k, v projection with A = O read through a tensor map over the
// layout attention left it in, and y stored as plain sequence-shard rows.
sp_status out_projection(const void *o, const void *w, const void *bias, void *y,
                         int32_t hidden, int32_t layout, const sp_shape *s, void *stream) {
  if (layout < SP_O_SEQ_SHARDED || layout > SP_O_RECV_CHUNKS) return SP_ERR_SHAPE;
  sp_status st = check_common(s, layout != SP_O_SEQ_SHARDED);
  if (st != SP_OK) return st;
  if (o == nullptr || w == nullptr || y == nullptr) return SP_ERR_NULL;
  if (hidden < 8 || hidden % 8 != 0) return SP_ERR_SHAPE;
  if (!aligned16(o) || !aligned16(w) || !aligned16(y) ||
      (bias != nullptr && (reinterpret_cast<uintptr_t>(bias) & 1u) != 0))
    return SP_ERR_ALIGN;
  const int P = s->P, B = s->B, H = s->H, D = s->D, N = s->N;
  const int Nl = (N + P - 1) / P, Np = Nl * P;
  const int Hl = H / P;
  const int64_t K = static_cast<int64_t>(H) * D;
  const int64_t rows = static_cast<int64_t>(layout == SP_O_RECV_CHUNKS ? 1 : P) * B * Nl;
  if (rows >= (int64_t(1) << 31) || rows * hidden >= (int64_t(1) << 40) ||
      static_cast<int64_t>(hidden) * K >= (int64_t(1) << 40))
    return SP_ERR_SHAPE;
  int32_t *status = status_ptr();
  if (status == nullptr) return SP_ERR_CUDA;
  CUtensorMap ma;
  sp::ProjParams p;
  std::memset(&p, 0, sizeof(p));
  const int64_t gcols = static_cast<int64_t>(Hl) * D;
  bool ok_a;
  int slots = 1;
  if (layout == SP_O_SEQ_SHARDED) {
    // [P][B][Nl][H][D] = rows x (H*D), row-major
    ok_a = make_map_rows4(&ma, o, K, rows, 1, 1, K, K * rows, K * rows, 128);
    p.a_load = sp::kALoadMatrix;
    p.rows_per_slot = static_cast<int32_t>(rows);
  } else if (layout == SP_O_HEAD_SHARDED) {
    // [P (group)][B][Np][Hl*D]: one slot per batch, rows = tokens of the slot
    ok_a = make_map_rows4(&ma, o, gcols, Np, B, P, gcols, gcols * Np, gcols * Np * B, 128);
    p.a_load = sp::kALoadHeads;
    p.rows_per_slot = Np;
    slots = B;
  } else {
    // one rank's [P (chunk)][B*Nl][Hl*D]
    ok_a = make_map_rows4(&ma, o, gcols, rows, P, 1, gcols, gcols * rows, gcols * rows * P, 128);
    p.a_load = sp::kALoadChunks;
    p.rows_per_slot = static_cast<int32_t>(rows);
  }
  if (!ok_a) return SP_ERR_CUDA;
  p.M = static_cast<int32_t>(rows);
  p.K = static_cast<int32_t>(K);
  p.nout = hidden;
  p.H = H;
  p.D = D;
  p.Hl = Hl;
  p.P = P;
  p.B = B;
  p.Nl = Nl;
  p.Np = Np;
  p.a_cols = static_cast<int32_t>(gcols);
  p.out_proj = 1;
  p.y = static_cast<__nv_bfloat16 *>(y);
  // with head groups and B > 1 a slot's rows are every B-th run of Nl rows
  p.tma_store = layout != SP_O_HEAD_SHARDED || B == 1;
  p.bias = static_cast<const __nv_bfloat16 *>(bias);
  p.status = status;
  return launch_projection(ma, w, slots, p, stream);
}

// Both projections: the tile counts for 256-row, 512-feature tiles, the map
// over w (a box of 128 rows: each CTA of a pair holds half of each 256-feature
// half of a tile), and
// the persistent launch on CTA pairs.  p holds every other field,
// rows_per_slot included.
sp_status launch_projection(const CUtensorMap &ma, const void *w, int slots, sp::ProjParams p,
                            void *stream) {
  p.tiles_per_slot = (p.rows_per_slot + sp::kPairBM - 1) / sp::kPairBM;
  const int64_t tiles_m = static_cast<int64_t>(p.tiles_per_slot) * slots;
  p.tiles_n = (p.nout + sp::kPairTileN - 1) / sp::kPairTileN;
  const int64_t tiles = tiles_m * p.tiles_n;
  if (tiles >= (int64_t(1) << 31)) return SP_ERR_SHAPE;
  p.tiles_m = static_cast<int32_t>(tiles_m);
  CUtensorMap mw;
  if (!make_map_matrix(&mw, w, p.K, p.nout, 128)) return SP_ERR_CUDA;
  CUtensorMap my[3] = {mw, mw, mw};   // unused unless the epilogue stores through TMA
  if (p.tma_store) {
    if (p.out_proj) {
      if (!make_map_out(&my[0], p.y, p.nout, p.M, 1)) return SP_ERR_CUDA;
    } else {
      const bool send = p.layout == sp::kProjSendChunks;
      const int64_t W = static_cast<int64_t>(send ? p.Hl : p.H) * p.D;
      for (int t = 0; t < 3; ++t)
        if (!make_map_out(&my[t], p.out[t], W, p.M, send ? p.P : 1)) return SP_ERR_CUDA;
    }
  }
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SP_ERR_CUDA;
  // persistent CTA pairs: as many clusters of two as can be resident at once
  // (or one per tile when there are fewer tiles)
  static bool attr_set[kMaxDevices] = {};
  static int max_pairs[kMaxDevices] = {};
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.blockDim = dim3(sp::kProjThreads);
  cfg.dynamicSmemBytes = sp::kPairSmemBytes;
  cfg.stream = cs;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  {
    std::lock_guard<std::mutex> g(g_mu);
    if (!attr_set[dev]) {
      if (cudaFuncSetAttribute(sp::projection_pair_kernel,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               sp::kPairSmemBytes) != cudaSuccess)
        return SP_ERR_CUDA;
      int sms = 0;
      if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return SP_ERR_CUDA;
      cfg.gridDim = dim3(static_cast<unsigned>(sms & ~1));
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, sp::projection_pair_kernel, &cfg) != cudaSuccess ||
          n < 1)
        return SP_ERR_CUDA;
      max_pairs[dev] = n;
      attr_set[dev] = true;
    }
  }
  const int64_t pairs = tiles < max_pairs[dev] ? tiles : max_pairs[dev];
  cfg.gridDim = dim3(static_cast<unsigned>(2 * pairs));
  cudaError_t e = cudaLaunchKernelEx(&cfg, sp::projection_pair_kernel, ma, mw, my[0], my[1], my[2], p);
  return launch_status(e == cudaSuccess ? cudaGetLastError() : e);
}

using AddressRangeFn = CUresult (*)(CUdeviceptr *, size_t *, CUdeviceptr);

AddressRangeFn address_range_fn() {
  static AddressRangeFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<AddressRangeFn>(p);
  });
  return fn;
}

// Source of the self-test's bulk copy (contents irrelevant).
__device__ __align__(128) uint8_t g_selftest_src[4096];

// The abort path of the kernels in miniature, on one warp: asynchronous work
// is in flight (a bulk copy into shared memory and one tcgen05 MMA into a
// TMEM accumulator) when a wait on a barrier that nothing completes runs out;
// the thread then drains what it issued (the copy's barrier, one more commit
// after the MMA) before the TMEM is released, and records SP_ERR_TIMEOUT.  A
// drain that did not finish, or a wait that did not run out, records a
// different code, so the caller sees it.
__global__ void __launch_bounds__(32, 1) wait_timeout_kernel(uint64_t limit_ns, int32_t *status) {
  __shared__ __align__(1024) uint8_t tiles[2 * 16384];  // A and B of one 128x128x16 MMA
  __shared__ __align__(128) uint8_t copy_dst[sizeof(g_selftest_src)];
  __shared__ __align__(8) uint64_t bars[3];              // never completed, copy, drain
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  const uint32_t never = sp::smem_u32(&bars[0]), copied = never + 8, drained = never + 16;
  if (threadIdx.x == 0) {
    sp::mbar_init(never, 1);
    sp::mbar_init(copied, 1);
    sp::mbar_init(drained, 1);
    abort_flag = 0;
    sp::fence_mbar_init();
  }
  __syncwarp();
  sp::tmem_alloc(sp::smem_u32(&tmem_slot), 128);
  sp::tmem_relinquish();
  sp::tc_fence_before();
  __syncwarp();
  sp::tc_fence_after();
  const uint32_t tmem = tmem_slot;
  if (threadIdx.x == 0) {
    sp::mbar_arrive_expect_tx(copied, sizeof(g_selftest_src));
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(sp::smem_u32(copy_dst)), "l"(reinterpret_cast<uint64_t>(g_selftest_src)),
          "r"(static_cast<uint32_t>(sizeof(g_selftest_src))), "r"(copied)
        : "memory");
    const uint32_t a = sp::smem_u32(tiles);
    sp::umma_ss<false>(tmem, sp::make_sdesc_sw128(a, 16, 1024),
                       sp::make_sdesc_sw128(a + 16384, 16, 1024),
                       sp::make_idesc_bf16(128, 128, 0, 0), 0u);
    // Nothing ever arrives on `never`: the wait must give up after limit_ns.
    const bool timed_out = !sp::mbar_wait(never, 0, &abort_flag, limit_ns);
    bool ok = sp::mbar_wait_drain(copied, 0, sp::kWaitLimitNs);
    sp::umma_commit(drained);
    ok = sp::mbar_wait_drain(drained, 0, sp::kWaitLimitNs) && ok;
    atomicExch(status, timed_out && ok ? sp::kStatusTimeout : sp::kStatusTimeout - 1);
  }
  sp::tc_fence_before();
  __syncwarp();
  sp::tc_fence_after();
  sp::tmem_dealloc(tmem, 128);
}

}  // namespace

extern "C" {

sp_status sp_selftest_wait_timeout(uint64_t limit_ns, void *stream) {
  NvtxRange range("sp_selftest_wait_timeout");
  if (limit_ns > 1000000000ull) limit_ns = 1000000000ull;
  int32_t *status = status_ptr();
  if (status == nullptr) return SP_ERR_CUDA;
  wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit_ns, status);
  return launch_status(cudaGetLastError());
}

int64_t sp_padded_tokens(int32_t N, int32_t P) {
  if (N < 1 || P < 1) return -1;
  return ((static_cast<int64_t>(N) + P - 1) / P) * P;
}

sp_status sp_check_shape(const sp_shape *shape) { return check_common(shape); }

sp_status sp_pack(const void *xs, void *xh, const sp_shape *shape, void *stream) {
  NvtxRange range("sp_pack");
  return permute(xs, xh, shape, stream, sp::kModePack);
}

sp_status sp_unpack(const void *oh, void *os, const sp_shape *shape, void *stream) {
  NvtxRange range("sp_unpack");
  return permute(oh, os, shape, stream, sp::kModeUnpack);
}

sp_status sp_shard(const void *x, void *xs, const sp_shape *shape, void *stream) {
  NvtxRange range("sp_shard");
  return permute(x, xs, shape, stream, sp::kModeShard);
}

sp_status sp_unshard(const void *xs, void *x, const sp_shape *shape, void *stream) {
  NvtxRange range("sp_unshard");
  return permute(xs, x, shape, stream, sp::kModeUnshard);
}

sp_status sp_exchange_pack(const void *xs_r, void *send, const sp_shape *shape, void *stream) {
  NvtxRange range("sp_exchange_pack");
  return permute(xs_r, send, shape, stream, sp::kModeExchangePack);
}

sp_status sp_exchange_unpack(const void *recv, void *os_r, const sp_shape *shape, void *stream) {
  NvtxRange range("sp_exchange_unpack");
  return permute(recv, os_r, shape, stream, sp::kModeExchangeUnpack);
}

sp_status sp_attention(const void *qh, const void *kh, const void *vh, void *oh, float *lse,
                       const sp_shape *shape, void *stream) {
  NvtxRange range("sp_attention");
  return attention(qh, kh, vh, oh, lse, shape, stream, false);
}

sp_status sp_attention_seqsharded(const void *qs, const void *ks, const void *vs, void *os,
                                  float *lse, const sp_shape *shape, void *stream) {
  NvtxRange range("sp_attention_seqsharded");
  return attention(qs, ks, vs, os, lse, shape, stream, true);
}

sp_status sp_attention_fp8_seqsharded(const void *qs, const void *ks, const void *vs,
                                      const float *q_scale, const float *k_scale,
                                      const float *v_scale, void *os, float *lse,
                                      const sp_shape *shape, void *stream) {
  NvtxRange range("sp_attention_fp8_seqsharded");
  if (q_scale == nullptr || k_scale == nullptr || v_scale == nullptr) return SP_ERR_NULL;
  return attention(qs, ks, vs, os, lse, shape, stream, true, q_scale, k_scale, v_scale);
}

sp_status sp_attention_sparse_seqsharded(const void *qs, const void *ks, const void *vs,
                                         const uint32_t *mask, void *os, float *lse,
                                         const sp_shape *shape, void *stream) {
  NvtxRange range("sp_attention_sparse_seqsharded");
  if (mask == nullptr) return SP_ERR_NULL;
  return attention(qs, ks, vs, os, lse, shape, stream, true, nullptr, nullptr, nullptr, mask);
}

sp_status sp_qkv_projection(const void *x, const void *w, const void *bias, void *q, void *k,
                            void *v, int32_t hidden, int32_t layout, const sp_shape *shape,
                            void *stream) {
  NvtxRange range("sp_qkv_projection");
  return qkv_projection(x, w, bias, q, k, v, hidden, layout, shape, stream);
}

sp_status sp_out_projection(const void *o, const void *w, const void *bias, void *y,
                            int32_t hidden, int32_t layout, const sp_shape *shape, void *stream) {
  NvtxRange range("sp_out_projection");
  return out_projection(o, w, bias, y, hidden, layout, shape, stream);
}

sp_status sp_attention_ulysses_peer(const void *const *q_shards, const void *k_group,
                                    const void *v_group, void *const *o_shards, float *lse,
                                    int32_t rank, const sp_shape *shape, void *stream) {
  NvtxRange range("sp_attention_ulysses_peer");
  return attention_peer(q_shards, k_group, v_group, o_shards, lse, rank, shape, stream);
}

sp_status sp_exchange_push(const void *k_r, const void *v_r, void *const *k_groups,
                           void *const *v_groups, uint64_t *const *counts, uint64_t epoch,
                           int32_t rank, const sp_shape *shape, void *stream) {
  NvtxRange range("sp_exchange_push");
  return exchange_push(k_r, v_r, k_groups, v_groups, counts, epoch, rank, shape, stream);
}

sp_status sp_attention_ulysses_overlap(const void *const *q_shards, const void *k_group,
                                       const void *v_group, void *const *o_shards, float *lse,
                                       const uint64_t *counts, uint64_t epoch, uint64_t wait_ns,
                                       int32_t rank, const sp_shape *shape, void *stream) {
  NvtxRange range("sp_attention_ulysses_overlap");
  if (counts == nullptr) return SP_ERR_NULL;
  if ((reinterpret_cast<uintptr_t>(counts) & 7u) != 0) return SP_ERR_ALIGN;
  if (epoch < 1) return SP_ERR_SHAPE;
  return attention_peer(q_shards, k_group, v_group, o_shards, lse, rank, shape, stream, counts,
                        epoch, wait_ns);
}

sp_status sp_ipc_export(const void *dev_ptr, void *handle_out, int64_t *offset_out) {
  if (dev_ptr == nullptr || handle_out == nullptr || offset_out == nullptr) return SP_ERR_NULL;
  AddressRangeFn range = address_range_fn();
  if (range == nullptr) return SP_ERR_CUDA;
  CUdeviceptr base = 0;
  size_t size = 0;
  if (range(&base, &size, reinterpret_cast<CUdeviceptr>(dev_ptr)) != CUDA_SUCCESS)
    return SP_ERR_CUDA;
  cudaIpcMemHandle_t h;
  if (cudaIpcGetMemHandle(&h, reinterpret_cast<void *>(base)) != cudaSuccess) return SP_ERR_CUDA;
  static_assert(sizeof(h) == SP_IPC_HANDLE_BYTES, "CUDA IPC handle size");
  std::memcpy(handle_out, &h, sizeof(h));
  *offset_out = static_cast<int64_t>(reinterpret_cast<CUdeviceptr>(dev_ptr) - base);
  return SP_OK;
}

sp_status sp_ipc_open(const void *handle, void **base_out) {
  if (handle == nullptr || base_out == nullptr) return SP_ERR_NULL;
  cudaIpcMemHandle_t h;
  std::memcpy(&h, handle, sizeof(h));
  if (cudaIpcOpenMemHandle(base_out, h, cudaIpcMemLazyEnablePeerAccess) != cudaSuccess)
    return SP_ERR_CUDA;
  return SP_OK;
}

sp_status sp_ipc_close(void *base) {
  if (base == nullptr) return SP_ERR_NULL;
  return cudaIpcCloseMemHandle(base) == cudaSuccess ? SP_OK : SP_ERR_CUDA;
}

sp_status sp_copy_heads(void *dst, int32_t dst_heads, int32_t dst_h0, const void *src,
                        int32_t src_heads, int32_t src_h0, int64_t rows, int32_t nh,
                        int32_t D, void *stream) {
  if (dst == nullptr || src == nullptr) return SP_ERR_NULL;
  if (rows < 0 || nh < 1 || D < 1 || dst_h0 < 0 || src_h0 < 0 ||
      static_cast<int64_t>(dst_h0) + nh > dst_heads || static_cast<int64_t>(src_h0) + nh > src_heads)
    return SP_ERR_SHAPE;
  const int64_t elt = sizeof(__nv_bfloat16);
  const int64_t dpitch = static_cast<int64_t>(dst_heads) * D * elt;
  const int64_t spitch = static_cast<int64_t>(src_heads) * D * elt;
  if (dpitch >= (int64_t{1} << 31) || spitch >= (int64_t{1} << 31)) return SP_ERR_SHAPE;
  if (rows == 0) return SP_OK;
  NvtxRange range("sp_copy_heads");
  char *d = static_cast<char *>(dst) + static_cast<int64_t>(dst_h0) * D * elt;
  const char *s = static_cast<const char *>(src) + static_cast<int64_t>(src_h0) * D * elt;
  const cudaError_t e = cudaMemcpy2DAsync(d, static_cast<size_t>(dpitch), s,
                                          static_cast<size_t>(spitch),
                                          static_cast<size_t>(nh) * D * elt,
                                          static_cast<size_t>(rows), cudaMemcpyDefault,
                                          static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? SP_OK : SP_ERR_CUDA;
}

sp_status sp_device_status(void *stream) {
  NvtxRange range("sp_device_status");
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  status_take_kernel<<<1, 1, 0, cs>>>();
  if (cudaGetLastError() != cudaSuccess) return SP_ERR_CUDA;
  int32_t v = 0;
  if (cudaMemcpyFromSymbolAsync(&v, g_status_taken, sizeof(v), 0, cudaMemcpyDeviceToHost, cs) !=
          cudaSuccess ||
      cudaStreamSynchronize(cs) != cudaSuccess)
    return SP_ERR_CUDA;
  if (v != 0) return v == sp::kStatusTimeout ? SP_ERR_TIMEOUT : SP_ERR_CUDA;
  return SP_OK;
}

uint64_t sp_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

const char *sp_status_str(sp_status status) {
  switch (status) {
    case SP_OK: return "ok";
    case SP_ERR_NULL: return "a required pointer is NULL";
    case SP_ERR_SHAPE: return "shape out of range";
    case SP_ERR_HEADS_NOT_DIVISIBLE: return "the degree P must divide the head count H";
    case SP_ERR_ALIGN: return "a device pointer is not 16-byte aligned";
    case SP_ERR_UNSUPPORTED_D: return "head dim D must be 64 or 128";
    case SP_ERR_CUDA: return "CUDA error";
    case SP_ERR_TIMEOUT: return "a kernel gave up on a bounded wait";
  }
  return "unknown status";
}

}  // extern "C"
