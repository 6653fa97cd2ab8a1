// Split-KV decode over an INT8 KV cache, plus the kernel that merges the splits.
//
// One query token per sequence attends to Skv cached keys whose K and V are stored as int8
// codes with one fp32 scale per (token, KV head).  The codes are used directly ("Flash
// Attention on Ascend: three techniques", section 3: the compressed cache takes part in the
// computation without being decompressed first):
//   score_j = scale * k_scale_j * (q . kcode_j)          O = sum_j p_j * v_scale_j * vcode_j
// so the scales leave the dot products and each code converts exactly to fp16.
//
// Split step (fa_decode_split_kernel): one CTA per (split, batch, KV head, block of <= 8 query
// heads of that KV head's group).  A producer warp streams the split's keys into a ring of
// shared-memory stages of 128 keys: the int8 K and V rows by TMA tensor copies (the codes never
// pass through registers on their way in, so the bytes in flight are bounded by shared memory,
// not by the register file), their fp32 scales by bulk copies (one per page or row segment;
// 4-byte asynchronous copies when a contiguous scale row is not 16-byte aligned), all
// completing on one mbarrier per stage.  Four consumer warps each take 32 keys of every stage, read the rows
// in their MMA fragment layout, convert the codes to fp16 with byte permutes and one fp16
// subtract, and run both contractions on the tensor cores with mma.sync m16n8k16 (fp32
// accumulate):
//   S  = Kcode[16 keys x 16 dims] . Q^T[16 dims x 8 heads]   (keys as M, heads as N)
//   O^T += Vcode^T[16 dims x 16 keys] . P'^T[16 keys x 8 heads]
// The reduction index of each contraction is permuted (dims for QK, dims of the output rows
// for PV) so that every thread's fragment comes from contiguous bytes of one row; Q and the
// output use the same permutations, so the results are unchanged.  P' = p * v_scale * 2^E is
// moved from the QK accumulator layout into the PV operand layout with movmatrix (8x8
// transpose); E keeps P' inside the fp16 range and is lowered, with an exact power-of-two
// rescale of the accumulator, whenever a larger v_scale arrives.  The online softmax (running
// max m and sum l per head, rescale when m grows by more than 2^8) runs on the accumulator
// fragments.  The 4 warps merge through shared memory and the CTA writes a normalised partial
// output and its log-sum-exp to the workspace.
//
// Paged variant (kPaged): the cache is a pool of pages of P keys (P a power of two >= 16),
// [num_pages, P, Hkv, D] codes and [num_pages, Hkv, P] scales, and sequence b owns the pages
// listed in block_table[b] ("Sparse attention and MLA operators in ops-transformer", section 2.2:
// the KV cache addressed through a block_table) and has its own length seqlens[b], read on the
// device ("Flash Attention on Ascend: three techniques", version section: sequences of different
// lengths in one batch).  The page becomes a TMA coordinate: a stage is min(128, P)-key boxes at
// (row in page, page id).  Splits are whole stages (ceil(len / splits) rounded up to 128 keys),
// so short sequences occupy few splits and the rest exit at once.  Page ids and lengths are
// range-checked; a bad one is recorded in the device status word and replaced by a valid one,
// so a corrupt table never makes the kernel read outside the pool.
//
// Merge step (fa_decode_combine_kernel): L = log sum_s exp(L_s), O = sum_s exp(L_s - L) O_s.
#pragma once

#include "sm100.cuh"

namespace fa {

// The paged kernel orders its CTAs by sequence length when the batch has at most this many
// sequences (one per thread of a CTA).
constexpr int kDecodeRankMaxB = 128;

struct DecodeParams {
  const uint16_t* q;  // bf16 [B, 1, Hq, D]
  const int8_t* k;    // [B, Skv, Hkv, D]; paged: [num_pages, P, Hkv, D]
  const int8_t* v;
  const float* k_scale;  // [B, Hkv, Skv]; paged: [num_pages, Hkv, P]
  const float* v_scale;
  float* o_part;    // [splits, B, Hq, D]
  float* lse_part;  // [splits, B, Hq]
  int B, Hq, Hkv, Skv, G, splits;
  float scale_log2;
  // paged cache only
  const int32_t* block_table;  // [B, max_pages]
  const int32_t* seqlens;      // [B]
  int max_pages, num_pages, page_shift;  // P = 1 << page_shift
};

struct CombineParams {
  const float* o_part;
  const float* lse_part;
  uint16_t* o;  // bf16 [B, 1, Hq, D]
  float* lse;   // [B, Hq] or null
  int B, Hq, splits;
};

// Two biased bytes (x + 128) in the low bytes of a fp16 pair with exponent 2^10 give
// 1024 + x + 128 exactly; subtracting 1152 leaves x exactly.
constexpr uint32_t kMagic64 = 0x64646464u;
__device__ __forceinline__ uint32_t f16x2_minus_1152(uint32_t h) {
  uint32_t d;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(h), "r"(0x64806480u));
  return d;
}
// bytes (x0, x1) at byte positions (lo, lo+1) of a biased word -> fp16x2 {x0, x1}
__device__ __forceinline__ uint32_t codes_to_f16x2(uint32_t biased, uint32_t sel) {
  return f16x2_minus_1152(prmt(biased, kMagic64, sel));
}
constexpr uint32_t kSelB01 = 0x4140u;  // [b0, 0x64, b1, 0x64]
constexpr uint32_t kSelB23 = 0x4342u;  // [b2, 0x64, b3, 0x64]

__device__ __forceinline__ void mma_f16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                              uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

// Power of two 2^e with e chosen so that x * 2^e < 2^top (x > 0), clamped to a safe range.
__device__ __forceinline__ int pow2_exponent_below(float x, int top) {
  if (!(x > 0.f)) return 0;
  int ex;
  frexpf(x, &ex);  // x = f * 2^ex, f in [0.5, 1): x < 2^ex
  return max(-100, min(100, top - ex));
}

__device__ __forceinline__ float exp2i(int e) { return __int_as_float((127 + e) << 23); }

__device__ __forceinline__ float exp2i_or_zero(int e) { return e < -126 ? 0.f : exp2i(e); }

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 r;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "r"(addr));
  return r;
}

__device__ __forceinline__ uint2 lds64(uint32_t addr) {
  uint2 r;
  asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(r.x), "=r"(r.y) : "r"(addr));
  return r;
}

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t r;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(r) : "r"(addr));
  return r;
}

__device__ __forceinline__ float lds32f(uint32_t addr) {
  float r;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(r) : "r"(addr));
  return r;
}

// 4-byte asynchronous global -> shared copy, and the mbarrier arrival that fires once every
// such copy of this thread has landed (the arrival raises the barrier's pending count when it
// is issued, so the phase cannot complete before the copies do).
__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_mbar_arrive(uint32_t bar) {
  asm volatile("cp.async.mbarrier.arrive.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}
// Bulk copy of `bytes` (a multiple of 16, both addresses 16-byte aligned) from global to shared
// memory, completing on `bar` (no multicast).
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes,
                                         uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(dst), "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}
// Announce `bytes` of asynchronous copies on `bar` without arriving on it.
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_all;" ::: "memory");
}

// Shape constants of the decode kernels.
constexpr int kDecodeStages = 2;      // K/V stages of 128 keys in the shared-memory ring (3 CTAs per SM)
constexpr int kDecodeMinChunk = 128;  // smallest split, in keys; a multiple of 128

// Shared-memory plan of the split kernel.  A stage holds 128 keys: the K and V code tiles
// ([128 rows][kRow bytes], swizzled like the TMA box so that the row-per-lane fragment reads
// spread over the banks) and their fp32 scales.
template <int D, int kBits>
struct DecodeCfg {
  static constexpr int kT = 128;                  // keys per stage
  static constexpr int kStages = kDecodeStages;
  static constexpr int kRow = D * kBits / 8;      // bytes of one key row of codes
  static constexpr int kTile = kT * kRow;         // bytes of one K or V code tile
  static constexpr int kStageBytes = 2 * kTile;
  static constexpr int kScaleOff = kStages * kStageBytes;  // fp32 [stages][K, V][kT]
  static constexpr int kBarOff = kScaleOff + kStages * 2 * kT * 4;
  static constexpr int kMiscOff = kBarOff + 16 * kStages;  // abort flag
  static constexpr int kPageStage = 256;                   // page ids staged per split
  static constexpr int kPageOff = kMiscOff + 16;
  static constexpr int kEnd = kPageOff + 4 * kPageStage;
  static constexpr int kSmemBytes = kEnd + 1024;           // + alignment of the dynamic base
  // merge buffers, reused from the stage tiles once the key loop is over
  static constexpr int kMergeO = 0;                        // fp32 [4 warps][8 heads][D]
  static constexpr int kMergeM = 4 * 8 * D * 4;            // fp32 [4][8]
  static constexpr int kMergeL = kMergeM + 4 * 8 * 4;      // fp32 [4][8]
  static_assert(kMergeL + 4 * 8 * 4 <= kScaleOff, "merge buffers must fit in the stage tiles");
};

// Byte offset in a code tile (base aligned to 1024 bytes) of byte `off` of the unswizzled tile:
// rows of 128 / 64 bytes use the TMA 128B / 64B swizzle (16-byte chunk index XOR address bits
// 7..9 / 7..8); 32-byte rows are stored plainly.
template <int kRow>
__device__ __forceinline__ uint32_t swz(uint32_t off) {
  if constexpr (kRow == 128) return off ^ (((off >> 7) & 7u) << 4);
  else if constexpr (kRow == 64) return off ^ (((off >> 7) & 3u) << 4);
  else return off;
}

// INT4 codes (4-bit two's complement) of a word -> fp16x2, exactly.  Flipping the top bit of a
// nibble gives its offset-binary value n = code + 8; the flip rides in the magic constant, so
// one logic op both masks and biases.  In fp16 with exponent 2^10 the mantissa counts units:
// nibbles at bits [0,4) and [16,20) give 1024 + n, minus 1032 leaves the code; nibbles at bits
// [4,8) and [20,24) give 1024 + 16 n, minus 1152 leaves 16 x the code (the caller folds 1/16
// into the other operand or the output).
__device__ __forceinline__ uint32_t nib_lo_f16x2(uint32_t raw) {
  const uint32_t h = (raw & 0x000F000Fu) ^ 0x64086408u;
  uint32_t d;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(h), "r"(0x64086408u));
  return d;
}
__device__ __forceinline__ uint32_t nib_hi16_f16x2(uint32_t raw) {
  const uint32_t h = (raw & 0x00F000F0u) ^ 0x64806480u;
  uint32_t d;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(h), "r"(0x64806480u));
  return d;
}

// 3 CTAs per SM for the 8-bit kernels (at most 136 registers a thread): the bytes in flight
// per SM set the decode's bandwidth.
template <int D, bool kPaged, int kBits>
__global__ void __launch_bounds__(160, kBits == 8 ? 3 : 1) fa_decode_split_kernel(
    const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
    const DecodeParams p) {
  using C = DecodeCfg<D, kBits>;
  constexpr int KS = D / 16;            // QK k-steps
  constexpr int MT = D / 16;            // PV m-tiles (16 output dims each)
  constexpr int QD = D / 4;             // QK: dims of each key row held by one thread
  constexpr int QW = QD * kBits / 32;   // ... as 32-bit words
  constexpr int DPT = D / 8;            // PV: output dims of one thread
  constexpr int VB = DPT * kBits / 8;   // ... as bytes of each V row
  constexpr int VW = (VB + 3) / 4;      // ... as 32-bit words
  // INT8 codes go to offset binary on load (the byte permutes need it); INT4 nibbles are biased
  // inside their conversion
  constexpr uint32_t kBias = kBits == 8 ? 0x80808080u : 0u;
  // the merge kernel may be scheduled as soon as every CTA of this grid has started
  asm volatile("griddepcontrol.launch_dependents;");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const uint32_t sb = smem_u32(smem);
  auto bar_full = [&](int s) { return sb + C::kBarOff + 8 * s; };
  auto bar_empty = [&](int s) { return sb + C::kBarOff + 8 * (C::kStages + s); };
  int* abort_flag = reinterpret_cast<int*>(smem + C::kMiscOff);
  int* sm_pages = reinterpret_cast<int*>(smem + C::kPageOff);
  const WaitCtl ctl{abort_flag, 4000000000ull};

  // grid (Hkv, splits, B * head blocks): the KV head varies fastest, so CTAs running at the
  // same time stream the same key rows (all KV heads of a key are contiguous in memory).
  const int kvh = blockIdx.x, split = blockIdx.y;
  const int nhb = (p.G + 7) / 8;
  int b = static_cast<int>(blockIdx.z) / nhb;
  const int hb = static_cast<int>(blockIdx.z) % nhb;
  if constexpr (kPaged) {
    // Longest sequences first: with mixed lengths a split's work is proportional to its
    // sequence's length, and CTAs start in grid order, so the long ones go in the first wave
    // rather than the last.  CTA rank r takes the sequence of length rank r (ties by index);
    // each thread ranks one sequence (up to kDecodeRankMaxB sequences; larger batches keep their
    // order).  Lengths are clamped as below, so a bad one cannot break the permutation.
    __shared__ int s_len[kDecodeRankMaxB];
    __shared__ int s_b;
    if (p.B <= kDecodeRankMaxB) {
      const int cap = p.max_pages << p.page_shift;
      if (threadIdx.x < p.B) s_len[threadIdx.x] = max(0, min(p.seqlens[threadIdx.x], cap));
      __syncthreads();
      if (threadIdx.x < p.B) {
        const int me = threadIdx.x, lme = s_len[me];
        int rank = 0;
        for (int x = 0; x < p.B; ++x) {
          const int lx = s_len[x];
          rank += (lx > lme || (lx == lme && x < me)) ? 1 : 0;
        }
        if (rank == b) s_b = me;
      }
      __syncthreads();
      b = s_b;
    }
  }
  const int head0 = kvh * p.G + hb * 8;
  const int nheads = min(8, p.G - hb * 8);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  int len = p.Skv;
  if constexpr (kPaged) {
    const int cap = p.max_pages << p.page_shift;
    len = p.seqlens[b];
    if (len < 0 || len > cap) {
      if (threadIdx.x == 0) atomicOr(&g_fa_device_status, kDevStatusBadIndex);
      len = max(0, min(len, cap));
    }
  }
  // splits are whole stages (every stage starts on a multiple of 128 keys) of at least
  // kDecodeMinChunk keys: a short sequence takes few splits rather than many tiny ones
  const int chunk = max(kDecodeMinChunk,
                        ((len + p.splits - 1) / p.splits + C::kT - 1) / C::kT * C::kT);
  const int t_begin = min(len, split * chunk);
  const int t_end = min(len, t_begin + chunk);
  const int n_stages = (t_end - t_begin + C::kT - 1) / C::kT;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(bar_full(s), 1);
      mbar_init(bar_empty(s), 4);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == 4) {
    // ============================ producer warp ============================
    const int pmask = (1 << p.page_shift) - 1;
    const int32_t* bt_row = kPaged ? p.block_table + static_cast<size_t>(b) * p.max_pages : nullptr;
    auto checked_page = [&](int slot) -> int {
      int pg = bt_row[slot];
      if (static_cast<unsigned>(pg) >= static_cast<unsigned>(p.num_pages)) {
        atomicOr(&g_fa_device_status, kDevStatusBadIndex);
        pg = 0;
      }
      return pg;
    };
    const int first_slot = kPaged ? (t_begin >> p.page_shift) : 0;
    const int n_slots = (kPaged && n_stages > 0) ? ((t_end - 1) >> p.page_shift) - first_slot + 1 : 0;
    const bool staged = n_slots <= C::kPageStage;
    if constexpr (kPaged) {
      if (staged)
        for (int i = lane; i < n_slots; i += 32) sm_pages[i] = checked_page(first_slot + i);
      __syncwarp();
    }
    // page of key t (t_begin <= t < t_end)
    auto page_of = [&](int t) -> int {
      const int slot = t >> p.page_shift;
      return staged ? sm_pages[slot - first_slot] : checked_page(slot);
    };
    const int box_t = kPaged ? min(C::kT, 1 << p.page_shift) : C::kT;  // keys per TMA box
    const float* ks_row = p.k_scale + (static_cast<size_t>(b) * p.Hkv + kvh) * p.Skv;
    const float* vs_row = p.v_scale + (static_cast<size_t>(b) * p.Hkv + kvh) * p.Skv;

    // scales by bulk copies whenever their rows are 16-byte aligned: page scale rows always
    // are (page_size >= 16); contiguous rows when Skv is a multiple of 4
    const bool bulk_scales = kPaged || (p.Skv % 4 == 0);
    // the K/V codes are read once per call: evict them first, so that streaming the cache does
    // not push the rest of a serving step's working set (a prefill's K/V, say) out of L2
    const uint64_t stream_pol = l2_evict_first_policy();
    int issued = 0;
    for (int i = 0; i < n_stages; ++i) {
      const int s = i % C::kStages;
      if (i >= C::kStages && !mbar_wait(bar_empty(s), ((i / C::kStages) - 1) & 1, ctl)) break;
      const int t0 = t_begin + C::kT * i;
      const uint32_t ks_dst = sb + C::kScaleOff + s * 2 * C::kT * 4;
      const uint32_t vs_dst = ks_dst + C::kT * 4;
      if (bulk_scales) {
        // One thread issues everything: the K/V code boxes and, beside each, its keys' scales
        // as one bulk copy (a page's scales are contiguous; so are a row segment's).  Keys past
        // the split's end get real scales of the same page or row; the consumers mask them.
        if (lane == 0) {
          const uint32_t seg =
              kPaged ? C::kT * 4 : static_cast<uint32_t>(min(C::kT, p.Skv - t0)) * 4;
          mbar_arrive_expect_tx(bar_full(s), C::kStageBytes + 2 * seg);
          const uint32_t kt = sb + s * C::kStageBytes, vt = kt + C::kTile;
          for (int t = t0; t < t0 + C::kT; t += box_t) {
            const uint32_t off = (t - t0) * C::kRow;  // box_t divides kT: stays inside the tile
            if constexpr (kPaged) {
              // a box past the split's last key reads the split's last page
              const int pg = page_of(min(t, t_end - 1));
              const int r0 = t & pmask;
              tma_load_4d_policy(kt + off, &tm_k, bar_full(s), 0, kvh, r0, pg, stream_pol);
              tma_load_4d_policy(vt + off, &tm_v, bar_full(s), 0, kvh, r0, pg, stream_pol);
              const size_t idx = ((static_cast<size_t>(pg) * p.Hkv + kvh) << p.page_shift) + r0;
              bulk_g2s(ks_dst + 4 * (t - t0), p.k_scale + idx, 4 * box_t, bar_full(s));
              bulk_g2s(vs_dst + 4 * (t - t0), p.v_scale + idx, 4 * box_t, bar_full(s));
            } else {
              tma_load_4d_policy(kt + off, &tm_k, bar_full(s), 0, kvh, t, b, stream_pol);
              tma_load_4d_policy(vt + off, &tm_v, bar_full(s), 0, kvh, t, b, stream_pol);
            }
          }
          if constexpr (!kPaged) {
            bulk_g2s(ks_dst, ks_row + t0, seg, bar_full(s));
            bulk_g2s(vs_dst, vs_row + t0, seg, bar_full(s));
          }
        }
        __syncwarp();
      } else {
        // Contiguous scale rows that are not 16-byte aligned: 4-byte asynchronous copies, 4 keys
        // per lane.  The K/V code tiles still go first: their byte count is announced without
        // an arrival, and the stage's one arrival comes only after every lane has registered
        // its scale copies, so the phase cannot complete early.
        if (lane == 0) {
          mbar_expect_tx(bar_full(s), C::kStageBytes);
          const uint32_t kt = sb + s * C::kStageBytes, vt = kt + C::kTile;
          for (int t = t0; t < t0 + C::kT; t += box_t) {
            const uint32_t off = (t - t0) * C::kRow;
            tma_load_4d_policy(kt + off, &tm_k, bar_full(s), 0, kvh, t, b, stream_pol);
            tma_load_4d_policy(vt + off, &tm_v, bar_full(s), 0, kvh, t, b, stream_pol);
          }
        }
#pragma unroll
        for (int j = 0; j < C::kT / 32; ++j) {
          const int r = lane + 32 * j, t = t0 + r;
          if (t < t_end) {
            cp_async4(ks_dst + 4 * r, ks_row + t);
            cp_async4(vs_dst + 4 * r, vs_row + t);
          }
        }
        cp_async_mbar_arrive(bar_full(s));  // each lane: +1 pending now, its arrival on completion
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_full(s));
      }
      issued = i + 1;
    }
    // Every copy this warp started has landed before the CTA can exit (already true on the
    // normal path; after a consumer gave up this waits, bounded, for copies in flight).
    cp_async_wait_all();
    if (lane == 0) {
      volatile int zero = 0;
      const WaitCtl drain_ctl{&zero, 4000000000ull};
      for (int s = 0; s < C::kStages && s < issued; ++s) {
        const int last = s + C::kStages * ((issued - 1 - s) / C::kStages);
        mbar_wait(bar_full(s), (last / C::kStages) & 1, drain_ctl);
      }
    }
    return;
  }

  // ============================ consumer warps 0..3 ============================
  const int g = lane >> 2, c = lane & 3;
  // Key of slot k (0..15) of a 16-key group, the same for the K rows (QK m-rows), their scales
  // and masks, and the V rows (PV k-index), so the product is unchanged.  4-bit code rows are 64
  // bytes: with the identity, the PV fragment reads of keys 2c (c = 0..3) would all fall in the
  // same half of their 128-byte lines (a 2-way bank conflict); flipping bit 0 when bit 1 is set
  // spreads them over both halves and both swizzle groups while keeping each QK pair (2i, 2i+1)
  // in different halves.
  auto kslot = [](int k) { return kBits == 4 ? (k ^ ((k >> 1) & 1)) : k; };

  // ---- Q as the B operand of the QK mma, fp16, scaled by 2^eq per head (exact) ----
  // Thread c holds dims [QD*c, QD*c + QD) of its head, in the order its K fragment takes them
  // from each key row: INT8 k-step s, element e is dim 4s + e of the block; INT4 k-step 2j + h
  // takes nibbles (2h, 2h+4) and (2h+1, 2h+5) of word j, i.e. dims 8j + 2h + {0, 4, 1, 5}.
  uint32_t qf[KS][2];
  float sc_mine;
  {
    float qv[KS][4];
    const bool hv = g < nheads;
    const uint16_t* qrow = p.q + (static_cast<size_t>(b) * p.Hq + head0 + (hv ? g : 0)) * D;
    float amax = 0.f;
#pragma unroll
    for (int s = 0; s < KS; ++s)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int dim = kBits == 8 ? 4 * s + e : 8 * (s >> 1) + 2 * (s & 1) + (e >> 1) + 4 * (e & 1);
        qv[s][e] = hv ? bf16_bits_to_float(qrow[QD * c + dim]) : 0.f;
        amax = fmaxf(amax, fabsf(qv[s][e]));
      }
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    const int eq = pow2_exponent_below(amax, 15);
    const float qs = exp2i(eq);
    // INT4: the K fragment's second pair of each k-step carries 16 x the code (nib_hi16), so
    // its Q partner is scaled by 1/16 (exact)
    const float qs_hi = kBits == 4 ? qs * 0.0625f : qs;
#pragma unroll
    for (int s = 0; s < KS; ++s) {
      qf[s][0] = pack_f16x2(qv[s][0] * qs, qv[s][1] * qs);
      qf[s][1] = pack_f16x2(qv[s][2] * qs_hi, qv[s][3] * qs_hi);
    }
    sc_mine = p.scale_log2 * exp2i(-eq);
  }
  // this thread's accumulator columns are heads 2c and 2c+1
  const float sc0 = __shfl_sync(0xffffffffu, sc_mine, 8 * c);
  const float sc1 = __shfl_sync(0xffffffffu, sc_mine, 8 * c + 4);

  float oacc[MT][4];
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) oacc[mt][0] = oacc[mt][1] = oacc[mt][2] = oacc[mt][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  // P' = p * v_scale * 2^E must stay below 2^15 in fp16 (p <= 2^8 with the lazy rescale): the
  // warp lowers E, rescaling its output accumulator, whenever a larger v_scale arrives.
  constexpr int kEUnset = 1 << 20;
  int E = kEUnset;

  for (int i = 0; i < n_stages; ++i) {
    const int s = i % C::kStages;
    if (!mbar_wait(bar_full(s), (i / C::kStages) & 1, ctl)) break;
    const int T = t_begin + C::kT * i + 32 * warp;  // this warp's 32 keys of the stage
    if (T < t_end) {
      const uint32_t kt = sb + s * C::kStageBytes, vt = kt + C::kTile;
      const uint32_t ks_s = sb + C::kScaleOff + s * 2 * C::kT * 4, vs_s = ks_s + C::kT * 4;
      const int r_w = 32 * warp;  // first row of this warp in the stage tiles

      // -- S = Kcode . Q^T per 16-key group; x = score in log2 units --
      float x[2][4];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        uint32_t kw[2][QW];  // this thread's words of rows g and g + 8 of the group
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
          const uint32_t row0 = (r_w + 16 * u + kslot(g + 8 * rr)) * C::kRow + QD * kBits / 8 * c;
#pragma unroll
          for (int w4 = 0; w4 < QW; w4 += 4) {
            if constexpr (QW >= 4) {
              const uint4 x = lds128(kt + swz<C::kRow>(row0 + 4 * w4));
              kw[rr][w4] = x.x ^ kBias;
              kw[rr][(w4 + 1) % QW] = x.y ^ kBias;
              kw[rr][(w4 + 2) % QW] = x.z ^ kBias;
              kw[rr][(w4 + 3) % QW] = x.w ^ kBias;
            } else {
              const uint2 x = lds64(kt + swz<C::kRow>(row0));
              kw[rr][0] = x.x ^ kBias;
              kw[rr][1 % QW] = x.y ^ kBias;
            }
          }
        }
        float sacc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int st = 0; st < KS; ++st) {
          if constexpr (kBits == 8) {
            const uint32_t w0 = kw[0][st], w1 = kw[1][st];
            mma_f16_16816(sacc, codes_to_f16x2(w0, kSelB01), codes_to_f16x2(w1, kSelB01),
                          codes_to_f16x2(w0, kSelB23), codes_to_f16x2(w1, kSelB23), qf[st][0],
                          qf[st][1]);
          } else {
            // k-step 2j + h of word j: nibbles (2h, 2h+4) as is, (2h+1, 2h+5) times 16
            const uint32_t w0 = kw[0][st >> 1] >> (8 * (st & 1));
            const uint32_t w1 = kw[1][st >> 1] >> (8 * (st & 1));
            mma_f16_16816(sacc, nib_lo_f16x2(w0), nib_lo_f16x2(w1), nib_hi16_f16x2(w0),
                          nib_hi16_f16x2(w1), qf[st][0], qf[st][1]);
          }
        }
        const int rA = r_w + 16 * u + kslot(g), rB = r_w + 16 * u + kslot(g + 8);
        const int tA = T + 16 * u + kslot(g), tB = T + 16 * u + kslot(g + 8);
        const float kA = lds32f(ks_s + 4 * rA), kB = lds32f(ks_s + 4 * rB);
        x[u][0] = tA < t_end ? sacc[0] * kA * sc0 : -INFINITY;
        x[u][1] = tA < t_end ? sacc[1] * kA * sc1 : -INFINITY;
        x[u][2] = tB < t_end ? sacc[2] * kB * sc0 : -INFINITY;
        x[u][3] = tB < t_end ? sacc[3] * kB * sc1 : -INFINITY;
      }

      // -- online softmax per head (columns 2c, 2c+1); max over the warp's 32 keys --
      float mx0 = fmaxf(fmaxf(x[0][0], x[0][2]), fmaxf(x[1][0], x[1][2]));
      float mx1 = fmaxf(fmaxf(x[0][1], x[0][3]), fmaxf(x[1][1], x[1][3]));
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
      }
      if (mx0 > m0 + 8.f) {
        const float a = ex2(m0 - mx0);
        m0 = mx0;
        l0 *= a;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          oacc[mt][0] *= a;
          oacc[mt][2] *= a;
        }
      }
      if (mx1 > m1 + 8.f) {
        const float a = ex2(m1 - mx1);
        m1 = mx1;
        l1 *= a;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          oacc[mt][1] *= a;
          oacc[mt][3] *= a;
        }
      }
      const float mu0 = (m0 == -INFINITY) ? 0.f : m0;
      const float mu1 = (m1 == -INFINITY) ? 0.f : m1;

      // -- value scales of the warp's keys; lower E if a larger one arrived --
      float vsc[2][2];
      float vmax = 0.f;
#pragma unroll
      for (int u = 0; u < 2; ++u)
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
          const int row = r_w + 16 * u + kslot(g + 8 * rr);
          vsc[u][rr] = (T + 16 * u + kslot(g + 8 * rr) < t_end) ? lds32f(vs_s + 4 * row) : 0.f;
          vmax = fmaxf(vmax, vsc[u][rr]);
        }
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
      const int e_step = pow2_exponent_below(vmax, 7);
      if (e_step < E) {
        if (E != kEUnset) {
          const float a = exp2i_or_zero(e_step - E);
#pragma unroll
          for (int mt = 0; mt < MT; ++mt) {
            oacc[mt][0] *= a;
            oacc[mt][1] *= a;
            oacc[mt][2] *= a;
            oacc[mt][3] *= a;
          }
        }
        E = e_step;
      }
      const float pscale = exp2i(E);

      uint32_t pb[2][2];  // PV B operand per group: keys 0-7 and 8-15 of the group
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const float pa0 = ex2(x[u][0] - mu0), pa1 = ex2(x[u][1] - mu1);
        const float pb0 = ex2(x[u][2] - mu0), pb1 = ex2(x[u][3] - mu1);
        l0 += pa0 + pb0;
        l1 += pa1 + pb1;
        const float wa = vsc[u][0] * pscale, wb = vsc[u][1] * pscale;
        pb[u][0] = movmatrix_trans(pack_f16x2(pa0 * wa, pa1 * wa));
        pb[u][1] = movmatrix_trans(pack_f16x2(pb0 * wb, pb1 * wb));
      }

      // -- O^T += Vcode^T . P'^T --
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        uint32_t r[4][VW];  // this thread's words of keys 2c, 2c+1, 2c+8, 2c+9 of the group
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          const int row = r_w + 16 * u + kslot(2 * c + (q4 & 1) + 8 * (q4 >> 1));
          const uint32_t off = swz<C::kRow>(row * C::kRow + VB * g);
          if constexpr (VB == 16) {
            const uint4 x = lds128(vt + off);
            r[q4][0] = x.x ^ kBias;
            r[q4][1 % VW] = x.y ^ kBias;
            r[q4][2 % VW] = x.z ^ kBias;
            r[q4][3 % VW] = x.w ^ kBias;
          } else if constexpr (VB == 8) {
            const uint2 x = lds64(vt + off);
            r[q4][0] = x.x ^ kBias;
            r[q4][1 % VW] = x.y ^ kBias;
          } else {
            r[q4][0] = lds32(vt + off) ^ kBias;
          }
        }
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          // output dims 2mt and 2mt+1 of this thread's block: INT8 bytes 2mt, 2mt+1; INT4 the
          // two nibbles of byte mt
          uint32_t a0, a1, a2, a3;
          if constexpr (kBits == 8) {
            const int w = mt >> 1;
            const uint32_t sel = (mt & 1) ? 0x7362u : 0x5140u;
            const uint32_t x01 = prmt(r[0][w], r[1][w], sel);  // keys 2c, 2c+1
            const uint32_t x89 = prmt(r[2][w], r[3][w], sel);  // keys 2c+8, 2c+9
            a0 = codes_to_f16x2(x01, kSelB01);
            a1 = codes_to_f16x2(x01, kSelB23);
            a2 = codes_to_f16x2(x89, kSelB01);
            a3 = codes_to_f16x2(x89, kSelB23);
          } else {
            const int w = mt >> 2;
            // byte mt & 3 of the first key's word into byte 0, of the second key's into byte 2
            constexpr uint32_t kSel[4] = {0x4400u, 0x5511u, 0x6622u, 0x7733u};
            const uint32_t x01 = prmt(r[0][w], r[1][w], kSel[mt & 3]);  // keys 2c, 2c+1
            const uint32_t x89 = prmt(r[2][w], r[3][w], kSel[mt & 3]);  // keys 2c+8, 2c+9
            // dim 2mt (low nibble) as is; dim 2mt+1 (high nibble) times 16, undone at the end
            a0 = nib_lo_f16x2(x01);
            a1 = nib_hi16_f16x2(x01);
            a2 = nib_lo_f16x2(x89);
            a3 = nib_hi16_f16x2(x89);
          }
          mma_f16_16816(oacc[mt], a0, a1, a2, a3, pb[u][0], pb[u][1]);
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(bar_empty(s));
  }

  // ---- merge the 4 warps (the stage tiles are free now: every stage has been consumed) ----
  named_bar_sync(1, 128);
  float* sm_o = reinterpret_cast<float*>(smem + C::kMergeO);
  float* sm_m = reinterpret_cast<float*>(smem + C::kMergeM);
  float* sm_l = reinterpret_cast<float*>(smem + C::kMergeL);
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, o);
    l1 += __shfl_xor_sync(0xffffffffu, l1, o);
  }
  if (g == 0) {
    sm_m[warp * 8 + 2 * c] = m0;
    sm_m[warp * 8 + 2 * c + 1] = m1;
    sm_l[warp * 8 + 2 * c] = l0;
    sm_l[warp * 8 + 2 * c + 1] = l1;
  }
  const float unscale = (E == kEUnset) ? 0.f : exp2i_or_zero(-E);
  // INT4: the odd dims (rows g + 8 of each m-tile) were accumulated from 16 x the codes
  const float unscale_hi = kBits == 4 ? unscale * 0.0625f : unscale;
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) {
    const int d0 = DPT * g + 2 * mt;
    float* ow = sm_o + warp * 8 * D;
    ow[(2 * c) * D + d0] = oacc[mt][0] * unscale;
    ow[(2 * c + 1) * D + d0] = oacc[mt][1] * unscale;
    ow[(2 * c) * D + d0 + 1] = oacc[mt][2] * unscale_hi;
    ow[(2 * c + 1) * D + d0 + 1] = oacc[mt][3] * unscale_hi;
  }
  named_bar_sync(1, 128);
  for (int idx = threadIdx.x; idx < nheads * D; idx += 128) {
    const int h = idx / D, d = idx % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < 4; ++w) M = fmaxf(M, sm_m[w * 8 + h]);
    float L = 0.f, acc = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const float mw = sm_m[w * 8 + h];
        const float f = (mw == -INFINITY) ? 0.f : ex2(mw - M);
        L += f * sm_l[w * 8 + h];
        acc += f * sm_o[(w * 8 + h) * D + d];
      }
    }
    const size_t row = (static_cast<size_t>(split) * p.B + b) * p.Hq + head0 + h;
    p.o_part[row * D + d] = (L > 0.f) ? acc / L : 0.f;
    if (d == 0) p.lse_part[row] = (L > 0.f) ? (M + __log2f(L)) * 0.69314718055994531f : -INFINITY;
  }
}

// One warp per (batch, query head): the lanes read the splits' log-sum-exps together, reduce
// the maximum and the sum of weights with shuffles, then each lane merges D/32 output dims with
// vector loads, several splits in flight at once.  Launched as a programmatic dependent of the
// split kernel: its CTAs may start while the split kernel drains and wait at griddepcontrol.wait
// until every partial is written and visible.
template <int D>
__global__ void __launch_bounds__(128) fa_decode_combine_kernel(const CombineParams p) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  constexpr int V = D / 32;  // dims per lane
  const int lane = threadIdx.x & 31;
  const int row = blockIdx.x * 4 + (threadIdx.x >> 5);
  const int rows = p.B * p.Hq;
  if (row >= rows) return;
  const size_t stride = static_cast<size_t>(rows);
  float M = -INFINITY;
  for (int s = lane; s < p.splits; s += 32) M = fmaxf(M, p.lse_part[s * stride + row]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  float L = 0.f;
  float acc[V];
#pragma unroll
  for (int i = 0; i < V; ++i) acc[i] = 0.f;
  if (M != -INFINITY) {
    for (int s = lane; s < p.splits; s += 32) {
      const float ls = p.lse_part[s * stride + row];
      L += (ls == -INFINITY) ? 0.f : expf(ls - M);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
#pragma unroll 4
    for (int s = 0; s < p.splits; ++s) {
      const float ls = p.lse_part[s * stride + row];
      const float w = (ls == -INFINITY) ? 0.f : expf(ls - M);
      const float* src = p.o_part + (s * stride + row) * D + V * lane;
      if constexpr (V == 4) {
        const float4 x = *reinterpret_cast<const float4*>(src);
        acc[0] += w * x.x;
        acc[1 % V] += w * x.y;
        acc[2 % V] += w * x.z;
        acc[3 % V] += w * x.w;
      } else {
        const float2 x = *reinterpret_cast<const float2*>(src);
        acc[0] += w * x.x;
        acc[1 % V] += w * x.y;
      }
    }
  }
  const float inv = (L > 0.f) ? 1.f / L : 0.f;
  uint16_t* dst = p.o + static_cast<size_t>(row) * D + V * lane;
  if constexpr (V == 4) {
    uint2 w2;
    w2.x = pack_bf16x2(acc[0] * inv, acc[1 % V] * inv);
    w2.y = pack_bf16x2(acc[2 % V] * inv, acc[3 % V] * inv);
    *reinterpret_cast<uint2*>(dst) = w2;
  } else {
    *reinterpret_cast<uint32_t*>(dst) = pack_bf16x2(acc[0] * inv, acc[1 % V] * inv);
  }
  if (lane == 0 && p.lse != nullptr) p.lse[row] = (L > 0.f) ? M + logf(L) : -INFINITY;
}

}  // namespace fa
