// Host side of libfa.so: argument validation, TMA descriptor encoding and kernel launches for
// the entry points declared in include/fa.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/fa.h"
#include "backward.cuh"
#include "decode.cuh"
#include "prefill.cuh"
#include "sm100.cuh"

// Scratch of the allocation-free decode entry point: one copy per GPU that loads the library,
// held until the process exits.  Shared by every call of fa_decode_int8_noalloc on that GPU.
static __device__ __align__(256) unsigned char g_noalloc_scratch[FA_DECODE_INT8_NOALLOC_MAX_SCRATCH];

namespace {

constexpr uint64_t kKernelTimeoutNs = 4000000000ull;  // bounded waits give up after 4 s

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// 4-D bf16 tensor [n3][n2][n1][n0] (n0 innermost), boxes of (64, b1, b2, 1), 128-byte swizzle.
int encode_bf16_4d(CUtensorMap* map, const void* base, uint64_t n0, uint64_t n1, uint64_t n2,
                   uint64_t n3, uint32_t b1, uint32_t b2) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return FA_ERR_CUDA;
  const cuuint64_t dims[4] = {n0, n1, n2, n3};
  const cuuint64_t strides[3] = {n0 * 2, n0 * n1 * 2, n0 * n1 * n2 * 2};
  const cuuint32_t box[4] = {64, b1, b2, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FA_OK : FA_ERR_CUDA;
}

// K or V codes viewed as a 4-D byte tensor (row bytes, Hkv, keys, B-or-pages); a box is
// `box_keys` key rows of one KV head.  Rows of 128 / 64 bytes are 128B / 64B-swizzled in shared
// memory, 32-byte rows are stored plainly.
int encode_u8_4d(CUtensorMap* map, const void* base, uint64_t n0, uint64_t n1, uint64_t n2,
                 uint64_t n3, uint32_t box_keys) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return FA_ERR_CUDA;
  const cuuint64_t dims[4] = {n0, n1, n2, n3};
  const cuuint64_t strides[3] = {n0, n0 * n1, n0 * n1 * n2};
  const cuuint32_t box[4] = {static_cast<cuuint32_t>(n0), 1, box_keys, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  n0 == 128  ? CU_TENSOR_MAP_SWIZZLE_128B
                  : n0 == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                             : CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FA_OK : FA_ERR_CUDA;
}

template <class Kernel>
int ensure_smem_attr(Kernel kernel, int bytes, std::atomic<uint64_t>& done_mask) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return FA_ERR_CUDA;
  const uint64_t bit = uint64_t(1) << dev;
  if (done_mask.load(std::memory_order_acquire) & bit) return FA_OK;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
      cudaSuccess)
    return FA_ERR_CUDA;
  done_mask.fetch_or(bit, std::memory_order_acq_rel);
  return FA_OK;
}

std::atomic<uint64_t> g_attr_prefill[8];
std::atomic<int> g_prefill_regs[8] = {};  // registers per thread of each variant, 0 = not read

// The optional parts of a forward call: an additive mask and global tokens.
struct PrefillExtra {
  const float* mask = nullptr;
  long long mask_sb = 0, mask_sh = 0;
  int n_global = 0;
};

template <int D, int kMode>
int launch_prefill(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                   int Hkv, int Sq, int Skv, float scale, int causal, int window,
                   const PrefillExtra& ex, cudaStream_t stream) {
  using C = fa::PrefillCfg<D>;
  fa::PrefillParams p{};
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.Sq = Sq;
  p.Skv = Skv;
  p.G = Hq / Hkv;
  p.Gp = 1;
  while (p.Gp < 8 && p.G % (2 * p.Gp) == 0) p.Gp *= 2;
  p.NP = p.G / p.Gp;
  const int tokens_per_cta = 256 / p.Gp;
  p.n_qblocks = (Sq + tokens_per_cta - 1) / tokens_per_cta;
  p.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  p.causal = causal;
  p.window = window;
  p.lse = lse;
  p.timeout_ns = kKernelTimeoutNs;
  p.mask = ex.mask;
  p.mask_sb = ex.mask_sb;
  p.mask_sh = ex.mask_sh;
  p.inv_scale = 1.0f / scale;
  p.mask_vec = (Skv % 4 == 0 && ex.mask_sb % 4 == 0 && ex.mask_sh % 4 == 0) ? 1 : 0;
  p.n_global = ex.n_global;

  const long long grid = static_cast<long long>(p.n_qblocks) * B * Hkv * p.NP;
  if (grid <= 0 || grid > 0x7fffffffLL) return FA_ERR_INVALID_ARG;

  CUtensorMap tq, tk, tv, to;
  const uint32_t tpt = 128 / p.Gp;
  int rc;
  if ((rc = encode_bf16_4d(&tq, q, D, Hq, Sq, B, p.Gp, tpt)) != FA_OK) return rc;
  if ((rc = encode_bf16_4d(&tk, k, D, Hkv, Skv, B, 1, 128)) != FA_OK) return rc;
  if ((rc = encode_bf16_4d(&tv, v, D, Hkv, Skv, B, 1, 128)) != FA_OK) return rc;
  if ((rc = encode_bf16_4d(&to, o, D, Hq, Sq, B, p.Gp, tpt)) != FA_OK) return rc;

  auto kernel = fa::fa_prefill_kernel<D, kMode>;
  const int variant = (D == 128 ? 4 : 0) + kMode;
  constexpr int smem_bytes = (kMode & fa::kModeMask) ? C::kSmemBytesMask : C::kSmemBytes;
  if ((rc = ensure_smem_attr(kernel, smem_bytes, g_attr_prefill[variant])) != FA_OK) return rc;
  // The kernel redistributes its launch registers between warpgroups (setmaxnreg); that only
  // completes if the launch gave every thread at least kMinLaunchRegs.
  int regs = g_prefill_regs[variant].load(std::memory_order_acquire);
  if (regs == 0) {
    cudaFuncAttributes attr;
    if (cudaFuncGetAttributes(&attr, kernel) != cudaSuccess) return FA_ERR_CUDA;
    regs = attr.numRegs;
    g_prefill_regs[variant].store(regs, std::memory_order_release);
  }
  if (regs < C::kMinLaunchRegs) return FA_ERR_UNSUPPORTED;
  kernel<<<static_cast<unsigned>(grid), C::kThreads, smem_bytes, stream>>>(tq, tk, tv, to, p);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

// fp32 [n2][n1][n0] array as a 3-D tensor; a box is `box0` consecutive elements of one row.
int encode_f32_3d(CUtensorMap* map, const void* base, uint64_t n0, uint64_t n1, uint64_t n2,
                  uint32_t box0) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return FA_ERR_CUDA;
  const cuuint64_t dims[3] = {n0, n1, n2};
  const cuuint64_t strides[2] = {n0 * 4, n0 * n1 * 4};
  const cuuint32_t box[3] = {box0, 1, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FA_OK : FA_ERR_CUDA;
}

// fp32 [n3][n2][n1][n0] (n0 innermost), boxes of (32, 1, 32, 1) = 32 rows of 128 bytes,
// 128-byte swizzle: the backward pass adds dQ tiles into its accumulator through it.
int encode_f32_4d_rows32(CUtensorMap* map, const void* base, uint64_t n0, uint64_t n1,
                         uint64_t n2, uint64_t n3) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return FA_ERR_CUDA;
  const cuuint64_t dims[4] = {n0, n1, n2, n3};
  const cuuint64_t strides[3] = {n0 * 4, n0 * n1 * 4, n0 * n1 * n2 * 4};
  const cuuint32_t box[4] = {32, 1, 32, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? FA_OK : FA_ERR_CUDA;
}

int bwd_sq_pad(int Sq) { return (Sq + 127) / 128 * 128; }

// -L log2(e) and -D per padded row, then the fp32 dQ accumulator [B, Sq, Hq, 128] (sized for
// the larger head dimension, so the size does not depend on D)
size_t bwd_ws_bytes(int B, int Hq, int Sq) {
  return 2ull * static_cast<size_t>(B) * Hq * bwd_sq_pad(Sq) * sizeof(float) +
         static_cast<size_t>(B) * Sq * Hq * 128 * sizeof(float);
}

std::atomic<uint64_t> g_attr_bwd[2];

template <int D>
int launch_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
               const float* lse, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int Sq,
               int Skv, float scale, int causal, int window, void* ws, cudaStream_t stream) {
  using C = fa::BwdCfg<D>;
  fa::BwdParams p{};
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.Sq = Sq;
  p.Skv = Skv;
  p.G = Hq / Hkv;
  p.Gp = 1;
  while (p.Gp < 8 && p.G % (2 * p.Gp) == 0) p.Gp *= 2;
  p.NP = p.G / p.Gp;
  p.Sq_pad = bwd_sq_pad(Sq);
  p.scale = scale;
  p.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  p.causal = causal;
  p.window = window;
  p.o = static_cast<const uint16_t*>(o);
  p.dout = static_cast<const uint16_t*>(dout);
  p.lse = lse;
  p.lse2 = static_cast<float*>(ws);
  p.delta = p.lse2 + static_cast<size_t>(B) * Hq * p.Sq_pad;
  p.dq_acc = p.delta + static_cast<size_t>(B) * Hq * p.Sq_pad;
  p.dq = static_cast<uint16_t*>(dq);
  p.timeout_ns = kKernelTimeoutNs;

  // 1. D and L * log2(e); the dQ accumulator zeroed
  const long long rows = static_cast<long long>(B) * Hq * p.Sq_pad;
  const long long rows_per_block = 8 * (256 / D);  // 8 warps of 256 / D rows each
  const long long prep_blocks = (rows + rows_per_block - 1) / rows_per_block;
  if (prep_blocks > 0x7fffffffLL) return FA_ERR_INVALID_ARG;
  fa::fa_bwd_prep_kernel<D><<<static_cast<unsigned>(prep_blocks), 256, 0, stream>>>(p);
  if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;

  int rc;
  CUtensorMap tk, tv, tq1, tdo1, tvec, tdk, tdv, tdqa;
  if ((rc = encode_bf16_4d(&tk, k, D, Hkv, Skv, B, 1, 128)) != FA_OK) return rc;
  if ((rc = encode_bf16_4d(&tv, v, D, Hkv, Skv, B, 1, 128)) != FA_OK) return rc;
  if ((rc = encode_bf16_4d(&tq1, q, D, Hq, Sq, B, 1, 128)) != FA_OK) return rc;
  if ((rc = encode_bf16_4d(&tdo1, dout, D, Hq, Sq, B, 1, 128)) != FA_OK) return rc;
  if ((rc = encode_f32_3d(&tvec, ws, p.Sq_pad, static_cast<uint64_t>(B) * Hq, 2, 128)) != FA_OK)
    return rc;
  if ((rc = encode_bf16_4d(&tdk, dk, D, Hkv, Skv, B, 1, 128)) != FA_OK) return rc;
  if ((rc = encode_bf16_4d(&tdv, dv, D, Hkv, Skv, B, 1, 128)) != FA_OK) return rc;
  if ((rc = encode_f32_4d_rows32(&tdqa, p.dq_acc, D, Hq, Sq, B)) != FA_OK) return rc;

  // 2. dK, dV and the dQ shares: one CTA per (b, KV head, key tile)
  p.n_tiles = (Skv + 127) / 128;
  const long long grid_kv = static_cast<long long>(p.n_tiles) * B * Hkv;
  if (grid_kv > 0x7fffffffLL) return FA_ERR_INVALID_ARG;
  auto kbwd = fa::fa_bwd_kernel<D>;
  if ((rc = ensure_smem_attr(kbwd, C::kUSmemBytes, g_attr_bwd[D == 128 ? 0 : 1])) != FA_OK)
    return rc;
  kbwd<<<static_cast<unsigned>(grid_kv), C::kThreads, C::kUSmemBytes, stream>>>(
      tq1, tk, tv, tdo1, tvec, tdk, tdv, tdqa, p);
  if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;

  // 3. dQ = scale * accumulator, bf16
  const long long n8 = static_cast<long long>(B) * Sq * Hq * D / 8;
  const long long fin_blocks = (n8 + 255) / 256;
  if (fin_blocks > 0x7fffffffLL) return FA_ERR_INVALID_ARG;
  fa::fa_bwd_dq_finalize_kernel<<<static_cast<unsigned>(fin_blocks), 256, 0, stream>>>(
      p.dq_acc, p.dq, scale, n8);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

size_t decode_ws_layout(int B, int Hq, int D, int splits, size_t* lse_off) {
  const size_t o_bytes = static_cast<size_t>(splits) * B * Hq * D * sizeof(float);
  const size_t off = (o_bytes + 255) & ~size_t(255);
  const size_t l_bytes = static_cast<size_t>(splits) * B * Hq * sizeof(float);
  if (lse_off) *lse_off = off;
  return (off + l_bytes + 255) & ~size_t(255);
}

// Fields every decode launch shares; the caller adds the cache addressing.
fa::DecodeParams decode_params(const void* q, const int8_t* k, const int8_t* v, const float* ks,
                               const float* vs, int B, int Hq, int Hkv, int D, float scale,
                               int splits, void* ws) {
  size_t lse_off = 0;
  decode_ws_layout(B, Hq, D, splits, &lse_off);
  fa::DecodeParams p{};
  p.q = static_cast<const uint16_t*>(q);
  p.k = k;
  p.v = v;
  p.k_scale = ks;
  p.v_scale = vs;
  p.o_part = static_cast<float*>(ws);
  p.lse_part = reinterpret_cast<float*>(static_cast<char*>(ws) + lse_off);
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.G = Hq / Hkv;
  p.splits = splits;
  p.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  return p;
}

std::atomic<uint64_t> g_attr_decode[8];

// Split kernel over grid (Hkv, splits, B * head blocks), then the merge kernel.  `keys` is the
// extent of the key axis of the code tensors (Skv, or the page size), `outer` that of the last
// axis (B, or the number of pages).
template <int D, bool kPaged, int kBits>
int launch_split_and_combine(const fa::DecodeParams& p, int keys, int outer, void* o, float* lse,
                             cudaStream_t stream) {
  using C = fa::DecodeCfg<D, kBits>;
  const long long gz = static_cast<long long>(p.B) * ((p.G + 7) / 8);
  if (p.splits > 65535 || gz > 65535) return FA_ERR_INVALID_ARG;
  CUtensorMap tk, tv;
  // a box is one stage (128 keys; past the end of the key axis TMA fills zeros and still counts
  // the bytes) or, for pages smaller than a stage, one page
  const uint32_t box = static_cast<uint32_t>(kPaged ? std::min(C::kT, keys) : C::kT);
  int rc;
  if ((rc = encode_u8_4d(&tk, p.k, C::kRow, p.Hkv, keys, outer, box)) != FA_OK) return rc;
  if ((rc = encode_u8_4d(&tv, p.v, C::kRow, p.Hkv, keys, outer, box)) != FA_OK) return rc;
  auto kernel = fa::fa_decode_split_kernel<D, kPaged, kBits>;
  const int variant = (D == 128 ? 4 : 0) + (kPaged ? 2 : 0) + (kBits == 4 ? 1 : 0);
  if ((rc = ensure_smem_attr(kernel, C::kSmemBytes, g_attr_decode[variant])) != FA_OK) return rc;
  dim3 grid(p.Hkv, p.splits, static_cast<unsigned>(gz));
  kernel<<<grid, 160, C::kSmemBytes, stream>>>(tk, tv, p);
  if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  fa::CombineParams cp{};
  cp.o_part = p.o_part;
  cp.lse_part = p.lse_part;
  cp.o = static_cast<uint16_t*>(o);
  cp.lse = lse;
  cp.B = p.B;
  cp.Hq = p.Hq;
  cp.splits = p.splits;
  // The merge is a programmatic dependent launch: its CTAs may be scheduled while the split
  // kernel drains, and wait on the device (griddepcontrol.wait) for the partials.
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>((static_cast<long long>(p.B) * p.Hq + 3) / 4));
  cfg.blockDim = dim3(128);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, fa::fa_decode_combine_kernel<D>, cp) != cudaSuccess)
    return FA_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

template <int D, int kBits>
int launch_decode(const void* q, const void* k, const void* v, const float* ks, const float* vs,
                  void* o, float* lse, int B, int Hq, int Hkv, int Skv, float scale, int splits,
                  void* ws, cudaStream_t stream) {
  fa::DecodeParams p = decode_params(q, static_cast<const int8_t*>(k),
                                     static_cast<const int8_t*>(v), ks, vs, B, Hq, Hkv, D, scale,
                                     splits, ws);
  p.Skv = Skv;
  return launch_split_and_combine<D, false, kBits>(p, Skv, B, o, lse, stream);
}

template <int D, int kBits>
int launch_decode_paged(const void* q, const void* k, const void* v, const float* ks,
                        const float* vs, const int32_t* block_table, const int32_t* seqlens,
                        void* o, float* lse, int B, int Hq, int Hkv, int page_shift,
                        int max_pages, int num_pages, float scale, int splits, void* ws,
                        cudaStream_t stream) {
  fa::DecodeParams p = decode_params(q, static_cast<const int8_t*>(k),
                                     static_cast<const int8_t*>(v), ks, vs, B, Hq, Hkv, D, scale,
                                     splits, ws);
  p.block_table = block_table;
  p.seqlens = seqlens;
  p.max_pages = max_pages;
  p.num_pages = num_pages;
  p.page_shift = page_shift;
  return launch_split_and_combine<D, true, kBits>(p, 1 << page_shift, num_pages, o, lse, stream);
}

// Device address of g_noalloc_scratch on the current device.  In host code the symbol name is
// only a host-side stand-in, so the address is looked up once per device, with that device
// current, and cached.
int noalloc_scratch_address(void** out) {
  static std::mutex mu;
  static void* addr[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return FA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr)
      return FA_ERR_CUDA;
    addr[dev] = p;
  }
  *out = addr[dev];
  return FA_OK;
}

__global__ void bounded_wait_selftest_kernel(uint64_t timeout_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    fa::mbar_init(fa::smem_u32(&bar), 1);
    fa::fence_mbar_init();
    const fa::WaitCtl ctl{&abort_flag, timeout_ns};
    // Nothing ever arrives on this barrier: the wait must give up on its own.
    fa::mbar_wait(fa::smem_u32(&bar), 0, ctl);
  }
}

// Argument checks shared by the contiguous decode entry points.
int check_decode(const void* q, const void* k, const void* v, const float* ks, const float* vs,
                 const void* o, const float* lse, int B, int Hq, int Hkv, int Skv, int D,
                 float scale, int num_splits) {
  if (!q || !k || !v || !ks || !vs || !o) return FA_ERR_INVALID_ARG;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Skv <= 0 || D <= 0 || num_splits <= 0)
    return FA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return FA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return FA_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(ks) ||
      !aligned16(vs) || (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)))
    return FA_ERR_ALIGNMENT;
  return FA_OK;
}

int check_workspace(int B, int Hq, int D, int num_splits, const void* ws, size_t ws_bytes) {
  if (!ws || ws_bytes < decode_ws_layout(B, Hq, D, num_splits, nullptr)) return FA_ERR_WORKSPACE;
  return aligned16(ws) ? FA_OK : FA_ERR_ALIGNMENT;
}

int decode_contiguous(int bits, const void* q, const void* k, const void* v, const float* ks,
                      const float* vs, void* o, float* lse, int B, int Hq, int Hkv, int Skv, int D,
                      float scale, int splits, void* ws, cudaStream_t s) {
  if (D == 128)
    return bits == 8 ? launch_decode<128, 8>(q, k, v, ks, vs, o, lse, B, Hq, Hkv, Skv, scale,
                                             splits, ws, s)
                     : launch_decode<128, 4>(q, k, v, ks, vs, o, lse, B, Hq, Hkv, Skv, scale,
                                             splits, ws, s);
  return bits == 8
             ? launch_decode<64, 8>(q, k, v, ks, vs, o, lse, B, Hq, Hkv, Skv, scale, splits, ws, s)
             : launch_decode<64, 4>(q, k, v, ks, vs, o, lse, B, Hq, Hkv, Skv, scale, splits, ws, s);
}

int decode_paged(int bits, const void* q, const void* k, const void* v, const float* ks,
                 const float* vs, const int32_t* block_table, const int32_t* seqlens, void* o,
                 float* lse, int B, int Hq, int Hkv, int page_size, int max_pages, int num_pages,
                 int D, float scale, int splits, void* ws, size_t ws_bytes, cudaStream_t st) {
  if (!q || !k || !v || !ks || !vs || !block_table || !seqlens || !o) return FA_ERR_INVALID_ARG;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || splits <= 0 || max_pages <= 0 || num_pages <= 0)
    return FA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return FA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return FA_ERR_INVALID_ARG;
  int shift = -1;
  for (int s = 4; s <= 16; ++s)
    if (page_size == (1 << s)) shift = s;
  if (shift < 0) return FA_ERR_INVALID_ARG;
  if ((static_cast<long long>(max_pages) << shift) > (1ll << 30)) return FA_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return FA_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(ks) ||
      !aligned16(vs) || (reinterpret_cast<uintptr_t>(block_table) & 3u) ||
      (reinterpret_cast<uintptr_t>(seqlens) & 3u) ||
      (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)))
    return FA_ERR_ALIGNMENT;
  const int rc = check_workspace(B, Hq, D, splits, ws, ws_bytes);
  if (rc != FA_OK) return rc;
  if (D == 128)
    return bits == 8 ? launch_decode_paged<128, 8>(q, k, v, ks, vs, block_table, seqlens, o, lse,
                                                   B, Hq, Hkv, shift, max_pages, num_pages,
                                                   scale, splits, ws, st)
                     : launch_decode_paged<128, 4>(q, k, v, ks, vs, block_table, seqlens, o, lse,
                                                   B, Hq, Hkv, shift, max_pages, num_pages,
                                                   scale, splits, ws, st);
  return bits == 8 ? launch_decode_paged<64, 8>(q, k, v, ks, vs, block_table, seqlens, o, lse, B,
                                                Hq, Hkv, shift, max_pages, num_pages, scale,
                                                splits, ws, st)
                   : launch_decode_paged<64, 4>(q, k, v, ks, vs, block_table, seqlens, o, lse, B,
                                                Hq, Hkv, shift, max_pages, num_pages, scale,
                                                splits, ws, st);
}

}  // namespace

extern "C" {

int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
           int Hkv, int Sq, int Skv, int D, float scale, int causal, int window, void* stream) {
  return fa_fwd_ext(q, k, v, o, lse, B, Hq, Hkv, Sq, Skv, D, scale, causal, window, 0, nullptr, 0,
                    0, stream);
}

int fa_fwd_ext(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
               int Hkv, int Sq, int Skv, int D, float scale, int causal, int window,
               int n_global, const float* mask, int64_t mask_batch_stride,
               int64_t mask_head_stride, void* stream) {
  if (!q || !k || !v || !o) return FA_ERR_INVALID_ARG;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Sq <= 0 || Skv <= 0 || D <= 0) return FA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return FA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
  if (window < 0 || (window > 0 && !causal)) return FA_ERR_INVALID_ARG;
  if (n_global < 0 || mask_batch_stride < 0 || mask_head_stride < 0) return FA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return FA_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) ||
      (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) ||
      (mask && (reinterpret_cast<uintptr_t>(mask) & 15u)))
    return FA_ERR_ALIGNMENT;
  PrefillExtra ex;
  ex.mask = mask;
  ex.mask_sb = mask_batch_stride;
  ex.mask_sh = mask_head_stride;
  ex.n_global = n_global;
  const int mode = (mask ? fa::kModeMask : 0) | (n_global > 0 ? fa::kModeGlobal : 0);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
#define FA_PREFILL_CASE(DD, MM)                                                                 \
  if (D == DD && mode == MM)                                                                   \
    return launch_prefill<DD, MM>(q, k, v, o, lse, B, Hq, Hkv, Sq, Skv, scale, causal, window, \
                                  ex, s);
  FA_PREFILL_CASE(128, 0)
  FA_PREFILL_CASE(128, 1)
  FA_PREFILL_CASE(128, 2)
  FA_PREFILL_CASE(128, 3)
  FA_PREFILL_CASE(64, 0)
  FA_PREFILL_CASE(64, 1)
  FA_PREFILL_CASE(64, 2)
  FA_PREFILL_CASE(64, 3)
#undef FA_PREFILL_CASE
  return FA_ERR_UNSUPPORTED;
}

size_t fa_bwd_workspace_bytes(int B, int Hq, int Sq) {
  if (B <= 0 || Hq <= 0 || Sq <= 0) return 0;
  return bwd_ws_bytes(B, Hq, Sq);
}

int fa_bwd(const void* q, const void* k, const void* v, const void* o, const void* dout,
           const float* lse, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int Sq,
           int Skv, int D, float scale, int causal, int window, void* workspace,
           size_t workspace_bytes, void* stream) {
  if (!q || !k || !v || !o || !dout || !lse || !dq || !dk || !dv) return FA_ERR_INVALID_ARG;
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || Sq <= 0 || Skv <= 0 || D <= 0) return FA_ERR_INVALID_ARG;
  if (Hq % Hkv != 0) return FA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
  if (window < 0 || (window > 0 && !causal)) return FA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return FA_ERR_UNSUPPORTED;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) ||
      !aligned16(dq) || !aligned16(dk) || !aligned16(dv) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u))
    return FA_ERR_ALIGNMENT;
  if (!workspace || workspace_bytes < bwd_ws_bytes(B, Hq, Sq)) return FA_ERR_WORKSPACE;
  if (!aligned16(workspace)) return FA_ERR_ALIGNMENT;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  return D == 128 ? launch_bwd<128>(q, k, v, o, dout, lse, dq, dk, dv, B, Hq, Hkv, Sq, Skv, scale,
                                    causal, window, workspace, s)
                  : launch_bwd<64>(q, k, v, o, dout, lse, dq, dk, dv, B, Hq, Hkv, Sq, Skv, scale,
                                   causal, window, workspace, s);
}

size_t fa_decode_int8_workspace_bytes(int B, int Hq, int D, int num_splits) {
  if (B <= 0 || Hq <= 0 || D <= 0 || num_splits <= 0) return 0;
  return decode_ws_layout(B, Hq, D, num_splits, nullptr);
}

const char* fa_status_string(int status) {
  switch (status) {
    case FA_OK: return "FA_OK";
    case FA_ERR_INVALID_ARG: return "FA_ERR_INVALID_ARG: invalid argument";
    case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED: unsupported head dimension";
    case FA_ERR_ALIGNMENT: return "FA_ERR_ALIGNMENT: pointer not 16-byte aligned";
    case FA_ERR_WORKSPACE: return "FA_ERR_WORKSPACE: workspace missing or too small";
    case FA_ERR_CUDA: return "FA_ERR_CUDA: CUDA call or kernel launch failed";
    case FA_ERR_TIMEOUT: return "FA_ERR_TIMEOUT: a kernel gave up a bounded wait";
    case FA_ERR_DEVICE_INDEX:
      return "FA_ERR_DEVICE_INDEX: a page id or sequence length in device memory was out of range";
    default: return "unknown fa_status";
  }
}

int fa_device_status(void* stream) {
  // One host thread at a time: the taken value passes through one device variable.
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  fa::status_take_kernel<<<1, 1, 0, s>>>();
  if (cudaGetLastError() != cudaSuccess) return FA_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return FA_ERR_CUDA;
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, fa::g_fa_status_taken, sizeof v) != cudaSuccess) return FA_ERR_CUDA;
  if (v == 0) return FA_OK;
  if (v & fa::kDevStatusTimeout) return FA_ERR_TIMEOUT;
  return (v & fa::kDevStatusBadIndex) ? FA_ERR_DEVICE_INDEX : FA_ERR_CUDA;
}

int fa_decode_int8(const void* q, const int8_t* k, const int8_t* v, const float* k_scale,
                   const float* v_scale, void* o, float* lse, int B, int Hq, int Hkv, int Skv,
                   int D, float scale, int num_splits, void* workspace, size_t workspace_bytes,
                   void* stream) {
  int rc = check_decode(q, k, v, k_scale, v_scale, o, lse, B, Hq, Hkv, Skv, D, scale, num_splits);
  if (rc == FA_OK) rc = check_workspace(B, Hq, D, num_splits, workspace, workspace_bytes);
  if (rc != FA_OK) return rc;
  return decode_contiguous(8, q, k, v, k_scale, v_scale, o, lse, B, Hq, Hkv, Skv, D, scale,
                           num_splits, workspace, static_cast<cudaStream_t>(stream));
}

int fa_decode_int4(const void* q, const uint8_t* k, const uint8_t* v, const float* k_scale,
                   const float* v_scale, void* o, float* lse, int B, int Hq, int Hkv, int Skv,
                   int D, float scale, int num_splits, void* workspace, size_t workspace_bytes,
                   void* stream) {
  int rc = check_decode(q, k, v, k_scale, v_scale, o, lse, B, Hq, Hkv, Skv, D, scale, num_splits);
  if (rc == FA_OK) rc = check_workspace(B, Hq, D, num_splits, workspace, workspace_bytes);
  if (rc != FA_OK) return rc;
  return decode_contiguous(4, q, k, v, k_scale, v_scale, o, lse, B, Hq, Hkv, Skv, D, scale,
                           num_splits, workspace, static_cast<cudaStream_t>(stream));
}

int fa_decode_int8_noalloc(const void* q, const int8_t* k, const int8_t* v, const float* k_scale,
                           const float* v_scale, void* o, float* lse, int B, int Hq, int Hkv,
                           int Skv, int D, float scale, int num_splits, void* stream) {
  int rc = check_decode(q, k, v, k_scale, v_scale, o, lse, B, Hq, Hkv, Skv, D, scale, num_splits);
  if (rc != FA_OK) return rc;
  if (decode_ws_layout(B, Hq, D, num_splits, nullptr) > FA_DECODE_INT8_NOALLOC_MAX_SCRATCH)
    return FA_ERR_WORKSPACE;
  void* ws = nullptr;
  if ((rc = noalloc_scratch_address(&ws)) != FA_OK) return rc;
  return decode_contiguous(8, q, k, v, k_scale, v_scale, o, lse, B, Hq, Hkv, Skv, D, scale,
                           num_splits, ws, static_cast<cudaStream_t>(stream));
}

int fa_decode_int8_paged(const void* q, const int8_t* k_pages, const int8_t* v_pages,
                         const float* k_scale_pages, const float* v_scale_pages,
                         const int32_t* block_table, const int32_t* seqlens, void* o, float* lse,
                         int B, int Hq, int Hkv, int page_size, int max_pages_per_seq,
                         int num_pages, int D, float scale, int num_splits, void* workspace,
                         size_t workspace_bytes, void* stream) {
  return decode_paged(8, q, k_pages, v_pages, k_scale_pages, v_scale_pages, block_table, seqlens,
                      o, lse, B, Hq, Hkv, page_size, max_pages_per_seq, num_pages, D, scale,
                      num_splits, workspace, workspace_bytes, static_cast<cudaStream_t>(stream));
}

int fa_decode_int4_paged(const void* q, const uint8_t* k_pages, const uint8_t* v_pages,
                         const float* k_scale_pages, const float* v_scale_pages,
                         const int32_t* block_table, const int32_t* seqlens, void* o, float* lse,
                         int B, int Hq, int Hkv, int page_size, int max_pages_per_seq,
                         int num_pages, int D, float scale, int num_splits, void* workspace,
                         size_t workspace_bytes, void* stream) {
  return decode_paged(4, q, k_pages, v_pages, k_scale_pages, v_scale_pages, block_table, seqlens,
                      o, lse, B, Hq, Hkv, page_size, max_pages_per_seq, num_pages, D, scale,
                      num_splits, workspace, workspace_bytes, static_cast<cudaStream_t>(stream));
}

int fa_selftest_bounded_wait(int timeout_us, void* stream) {
  if (timeout_us < 1 || timeout_us > 10000000) return FA_ERR_INVALID_ARG;
  bounded_wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<uint64_t>(timeout_us) * 1000ull);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

}  // extern "C"
