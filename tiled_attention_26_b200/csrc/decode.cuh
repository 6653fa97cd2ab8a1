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
// heads of that KV head's group); 4 warps stride over the split's keys 32 at a time.  Each warp
// streams the int8 rows straight from HBM into registers with 16-byte non-caching loads,
// converts them to fp16 with byte permutes and one fp16 subtract, and runs both contractions on
// the tensor cores with mma.sync m16n8k16 (fp32 accumulate):
//   S  = Kcode[16 tokens x 16 dims] . Q^T[16 dims x 8 heads]   (tokens as M, heads as N)
//   O^T += Vcode^T[16 dims x 16 tokens] . P'^T[16 tokens x 8 heads]
// The reduction index of each contraction is permuted (dims for QK, dims of the output rows
// for PV) so that every thread's fragment comes from contiguous bytes of one row; Q and the
// output use the same permutations, so the results are unchanged.  P' = p * v_scale is moved
// from the QK accumulator layout into the PV operand layout with movmatrix (8x8 transpose).
// The online softmax (running max m and sum l per head, rescale when m grows by more than 2^8)
// runs on the accumulator fragments.  The 4 warps merge through shared memory and the CTA
// writes a normalised partial output and its log-sum-exp to the workspace.
//
// Paged variant (kPaged): the cache is a pool of pages of P tokens (P a power of two >= 16),
// [num_pages, P, Hkv, D] codes and [num_pages, Hkv, P] scales, and sequence b owns the pages
// listed in block_table[b] ("Sparse attention and MLA operators in ops-transformer", section 2.2:
// the KV cache addressed through a block_table) and has its own length seqlens[b], read on the
// device ("Flash Attention on Ascend: three techniques", version section: sequences of different
// lengths in one batch).  Each split covers ceil(len / splits) keys rounded up to 16, so every
// 16-token group of a step lies inside one page: the page is looked up once per group.  Page ids
// and lengths are range-checked; a bad one is recorded in the device status word and replaced by
// a valid one, so a corrupt table never makes the kernel read outside the pool.
//
// Merge step (fa_decode_combine_kernel): L = log sum_s exp(L_s), O = sum_s exp(L_s - L) O_s.
#pragma once

#include "sm100.cuh"

namespace fa {

struct DecodeParams {
  const uint16_t* q;  // bf16 [B, 1, Hq, D]
  const int8_t* k;    // [B, Skv, Hkv, D]; paged: [num_pages, P, Hkv, D]
  const int8_t* v;
  const float* k_scale;  // [B, Hkv, Skv]; paged: [num_pages, Hkv, P]
  const float* v_scale;
  float* o_part;    // [splits, B, Hq, D]
  float* lse_part;  // [splits, B, Hq]
  int B, Hq, Hkv, Skv, G, splits, chunk;
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

__device__ __forceinline__ uint4 ldg_stream16(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__device__ __forceinline__ uint2 ldg_stream8(const void* p) {
  uint2 r;
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];"
               : "=r"(r.x), "=r"(r.y)
               : "l"(p));
  return r;
}

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

#ifndef FA_PAGED_SMEM_PAGES
#define FA_PAGED_SMEM_PAGES 1  // stage each split's page ids in shared memory
#endif

#ifndef FA_PAGED_VMAX_BATCH
#define FA_PAGED_VMAX_BATCH 1
#endif

#ifndef FA_DECODE_PDL
#define FA_DECODE_PDL 1  // launch the merge kernel as a programmatic dependent of the split kernel
#endif

#ifndef FA_DECODE_MIN_CTAS
#define FA_DECODE_MIN_CTAS 3  // CTAs per SM the register allocation must allow
#endif

template <int D, bool kPaged>
__global__ void __launch_bounds__(128, FA_DECODE_MIN_CTAS) fa_decode_split_kernel(const DecodeParams p) {
  constexpr int KS = D / 16;  // QK k-steps
  constexpr int MT = D / 16;  // PV m-tiles (16 output dims each)
  constexpr int VB = D / 8;   // V bytes per thread per token
  // grid (Hkv, splits, B * head blocks): the KV head varies fastest, so CTAs running at the
  // same time stream the same token rows (all KV heads of a token are contiguous in memory).
  // the merge kernel may be scheduled as soon as every CTA of this grid has started
  asm volatile("griddepcontrol.launch_dependents;");
  const int kvh = blockIdx.x, split = blockIdx.y;
  const int nhb = (p.G + 7) / 8;
  const int b = static_cast<int>(blockIdx.z) / nhb, hb = static_cast<int>(blockIdx.z) % nhb;
  const int head0 = kvh * p.G + hb * 8;
  const int nheads = min(8, p.G - hb * 8);
  int len = p.Skv, chunk = p.chunk;
  const int32_t* bt_row = nullptr;
  if constexpr (kPaged) {
    const int cap = p.max_pages << p.page_shift;
    len = p.seqlens[b];
    if (len < 0 || len > cap) {
      if (threadIdx.x == 0) atomicOr(&g_fa_device_status, kDevStatusBadIndex);
      len = max(0, min(len, cap));
    }
    chunk = ((len + p.splits - 1) / p.splits + 15) & ~15;
    bt_row = p.block_table + static_cast<size_t>(b) * p.max_pages;
  }
  const int t_begin = split * chunk;
  const int t_end = min(len, t_begin + chunk);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;

  __shared__ float sm_red[4];
  __shared__ float sm_m[4][8], sm_l[4][8];
  __shared__ float sm_o[4][8][D];

  const size_t row_stride = static_cast<size_t>(p.Hkv) * D;  // bytes between tokens
  const int pmask = (1 << p.page_shift) - 1;
  // physical page of key t (t < len): checked against the pool, never outside it
  auto checked_page = [&](int slot) -> int {
    int pg = bt_row[slot];
    if (static_cast<unsigned>(pg) >= static_cast<unsigned>(p.num_pages)) {
      atomicOr(&g_fa_device_status, kDevStatusBadIndex);
      pg = 0;
    }
    return pg;
  };
#if FA_PAGED_SMEM_PAGES
  // The split's page ids are staged in shared memory once (checked there), so the loads of a
  // step never wait on a dependent global load.  A split spanning more pages than the stage
  // holds reads the table directly.
  constexpr int kPageStage = 512;
  __shared__ int sm_pages[kPageStage];
  const int first_slot = kPaged ? (t_begin >> p.page_shift) : 0;
  const int n_slots = (kPaged && t_end > t_begin) ? ((t_end - 1) >> p.page_shift) - first_slot + 1 : 0;
  const bool staged = n_slots <= kPageStage;
  if constexpr (kPaged) {
    if (staged)
      for (int i = threadIdx.x; i < n_slots; i += 128) sm_pages[i] = checked_page(first_slot + i);
    __syncthreads();
  }
  auto page_of = [&](int t) -> int {
    const int slot = t >> p.page_shift;
    return staged ? sm_pages[slot - first_slot] : checked_page(slot);
  };
#else
  auto page_of = [&](int t) -> int { return checked_page(t >> p.page_shift); };
#endif
  // offset of (page pg, kv head kvh, row r) in the [num_pages, Hkv, P] scale arrays
  auto page_scale_index = [&](int pg, int r) -> size_t {
    return ((static_cast<size_t>(pg) * p.Hkv + kvh) << p.page_shift) + r;
  };
  // paged: code row and scale pointers of the 16-token group that starts at key gs0.  A group
  // past the split's last key is replaced by the split's last group (its extra keys are masked),
  // so every page looked up belongs to this split.
  const int last16 = (t_end - 1) & ~15;
  auto group_base = [&](int gs0, const int8_t* codes, const float* scales, const int8_t*& rows,
                        const float*& sc) {
    const int gs = min(gs0, last16);
    const int pg = page_of(gs);
    const int r0 = gs & pmask;
    rows = codes + ((static_cast<size_t>(pg) << p.page_shift) + r0) * row_stride +
           static_cast<size_t>(kvh) * D;
    sc = scales + page_scale_index(pg, r0);
  };

  const float* ks_row = p.k_scale + (static_cast<size_t>(b) * p.Hkv + kvh) * p.Skv;
  const float* vs_row = p.v_scale + (static_cast<size_t>(b) * p.Hkv + kvh) * p.Skv;

  // ---- P' = p * v_scale * 2^E stays below 2^15 in fp16: E from the split's largest v_scale ----
  float vmax = 0.f;
  if constexpr (kPaged) {
#if FA_PAGED_VMAX_BATCH
    // 8 keys per thread per round: all page ids, then all scales, so each round waits for two
    // memory latencies instead of sixteen
    for (int t0 = t_begin + threadIdx.x; t0 < t_end; t0 += 128 * 8) {
      int pg[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int t = min(t0 + 128 * i, t_end - 1);
        pg[i] = page_of(t);
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int t = t0 + 128 * i;
        const float sv = p.v_scale[page_scale_index(pg[i], min(t, t_end - 1) & pmask)];
        vmax = fmaxf(vmax, sv);
      }
    }
#else
    for (int t = t_begin + threadIdx.x; t < t_end; t += 128)
      vmax = fmaxf(vmax, p.v_scale[page_scale_index(page_of(t), t & pmask)]);
#endif
  } else {
    for (int t = t_begin + threadIdx.x; t < t_end; t += 128) vmax = fmaxf(vmax, vs_row[t]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
  if (lane == 0) sm_red[warp] = vmax;
  __syncthreads();
  vmax = fmaxf(fmaxf(sm_red[0], sm_red[1]), fmaxf(sm_red[2], sm_red[3]));
  const int E = pow2_exponent_below(vmax, 7);  // p <= 2^8 with the lazy rescale
  const float pscale = exp2i(E);

  // ---- Q as the B operand of the QK mma, fp16, scaled by 2^eq per head (exact) ----
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
        const int dim = (s / 4) * 64 + 16 * c + 4 * (s % 4) + e;
        qv[s][e] = hv ? bf16_bits_to_float(qrow[dim]) : 0.f;
        amax = fmaxf(amax, fabsf(qv[s][e]));
      }
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    const int eq = pow2_exponent_below(amax, 15);
    const float qs = exp2i(eq);
#pragma unroll
    for (int s = 0; s < KS; ++s) {
      qf[s][0] = pack_f16x2(qv[s][0] * qs, qv[s][1] * qs);
      qf[s][1] = pack_f16x2(qv[s][2] * qs, qv[s][3] * qs);
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

  const int8_t* kbase = p.k + (static_cast<size_t>(b) * p.Skv * p.Hkv + kvh) * D;
  const int8_t* vbase = p.v + (static_cast<size_t>(b) * p.Skv * p.Hkv + kvh) * D;
  const int nsteps = (t_end - t_begin + 31) / 32;

  // Each warp takes every 4th 32-token step.  Loads run one step ahead without extra registers:
  // the next step's K rows are requested as soon as this step's QK^T has consumed the K
  // registers, the next step's V rows as soon as PV has consumed the V registers.
  uint32_t kw[2][2][KS];  // [group][row g / g+8][k-step]
  uint32_t vw[2][4][VB / 4];
  float ksc[2][2], vsc[2][2];
  auto load_k = [&](int T) {
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int8_t* gk = nullptr;
      const float* gks = nullptr;
      if constexpr (kPaged) group_base(T + 16 * u, p.k, p.k_scale, gk, gks);
#pragma unroll
      for (int rr = 0; rr < 2; ++rr) {
        const int tok = min(T + 16 * u + g + 8 * rr, len - 1);
        const int8_t* row = kPaged ? gk + static_cast<size_t>(g + 8 * rr) * row_stride
                                   : kbase + static_cast<size_t>(tok) * row_stride;
        const uint4 lo = ldg_stream16(row + 16 * c);
        kw[u][rr][0] = lo.x;
        kw[u][rr][1] = lo.y;
        kw[u][rr][2] = lo.z;
        kw[u][rr][3] = lo.w;
        if constexpr (D == 128) {
          const uint4 hi = ldg_stream16(row + 64 + 16 * c);
          kw[u][rr][4 % KS] = hi.x;
          kw[u][rr][5 % KS] = hi.y;
          kw[u][rr][6 % KS] = hi.z;
          kw[u][rr][7 % KS] = hi.w;
        }
        ksc[u][rr] = kPaged ? gks[g + 8 * rr] : ks_row[tok];
      }
    }
  };
  auto load_v = [&](int T) {
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int8_t* gv = nullptr;
      const float* gvs = nullptr;
      if constexpr (kPaged) group_base(T + 16 * u, p.v, p.v_scale, gv, gvs);
#pragma unroll
      for (int rr = 0; rr < 2; ++rr)
        vsc[u][rr] = kPaged ? gvs[g + 8 * rr] : vs_row[min(T + 16 * u + g + 8 * rr, len - 1)];
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        const int off = 2 * c + (q4 & 1) + 8 * (q4 >> 1);
        const int tok = min(T + 16 * u + off, len - 1);
        const int8_t* row = (kPaged ? gv + static_cast<size_t>(off) * row_stride
                                    : vbase + static_cast<size_t>(tok) * row_stride) +
                            VB * g;
        if constexpr (VB == 16) {
          const uint4 x = ldg_stream16(row);
          vw[u][q4][0] = x.x;
          vw[u][q4][1 % (VB / 4)] = x.y;
          vw[u][q4][2 % (VB / 4)] = x.z;
          vw[u][q4][3 % (VB / 4)] = x.w;
        } else {
          const uint2 x = ldg_stream8(row);
          vw[u][q4][0] = x.x;
          vw[u][q4][1 % (VB / 4)] = x.y;
        }
      }
    }
  };
  if (warp < nsteps) {
    load_k(t_begin + 32 * warp);
    load_v(t_begin + 32 * warp);
  }
  for (int st = warp; st < nsteps; st += 4) {
    const int T = t_begin + 32 * st;
    const bool has_next = st + 4 < nsteps;

    // -- S = Kcode . Q^T per 16-token group; x = score in log2 units --
    float x[2][4];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      float sacc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int s = 0; s < KS; ++s) {
        const uint32_t w0 = kw[u][0][s] ^ 0x80808080u, w1 = kw[u][1][s] ^ 0x80808080u;
        mma_f16_16816(sacc, codes_to_f16x2(w0, kSelB01), codes_to_f16x2(w1, kSelB01),
                      codes_to_f16x2(w0, kSelB23), codes_to_f16x2(w1, kSelB23), qf[s][0],
                      qf[s][1]);
      }
      const int tA = T + 16 * u + g, tB = tA + 8;
      x[u][0] = tA < t_end ? sacc[0] * ksc[u][0] * sc0 : -INFINITY;
      x[u][1] = tA < t_end ? sacc[1] * ksc[u][0] * sc1 : -INFINITY;
      x[u][2] = tB < t_end ? sacc[2] * ksc[u][1] * sc0 : -INFINITY;
      x[u][3] = tB < t_end ? sacc[3] * ksc[u][1] * sc1 : -INFINITY;
    }
    if (has_next) load_k(T + 128);

    // -- online softmax per head (columns 2c, 2c+1); max over the warp's 32 tokens --
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
    uint32_t pb[2][2];  // PV B operand per group: tokens 0-7 and 8-15 of the group
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
      uint32_t r[4][VB / 4];
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4)
#pragma unroll
        for (int w = 0; w < VB / 4; ++w) r[q4][w] = vw[u][q4][w] ^ 0x80808080u;
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        const int w = mt >> 1;
        const uint32_t sel = (mt & 1) ? 0x7362u : 0x5140u;
        const uint32_t x01 = prmt(r[0][w], r[1][w], sel);  // tokens 2c, 2c+1
        const uint32_t x89 = prmt(r[2][w], r[3][w], sel);  // tokens 2c+8, 2c+9
        mma_f16_16816(oacc[mt], codes_to_f16x2(x01, kSelB01), codes_to_f16x2(x01, kSelB23),
                      codes_to_f16x2(x89, kSelB01), codes_to_f16x2(x89, kSelB23), pb[u][0],
                      pb[u][1]);
      }
    }
    if (has_next) load_v(T + 128);
  }

  // ---- merge the 4 warps ----
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, o);
    l1 += __shfl_xor_sync(0xffffffffu, l1, o);
  }
  if (g == 0) {
    sm_m[warp][2 * c] = m0;
    sm_m[warp][2 * c + 1] = m1;
    sm_l[warp][2 * c] = l0;
    sm_l[warp][2 * c + 1] = l1;
  }
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) {
    const int d0 = VB * g + 2 * mt;
    sm_o[warp][2 * c][d0] = oacc[mt][0];
    sm_o[warp][2 * c + 1][d0] = oacc[mt][1];
    sm_o[warp][2 * c][d0 + 1] = oacc[mt][2];
    sm_o[warp][2 * c + 1][d0 + 1] = oacc[mt][3];
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < nheads * D; idx += 128) {
    const int h = idx / D, d = idx % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < 4; ++w) M = fmaxf(M, sm_m[w][h]);
    float L = 0.f, acc = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const float f = (sm_m[w][h] == -INFINITY) ? 0.f : ex2(sm_m[w][h] - M);
        L += f * sm_l[w][h];
        acc += f * sm_o[w][h][d];
      }
    }
    const size_t row = (static_cast<size_t>(split) * p.B + b) * p.Hq + head0 + h;
    p.o_part[row * D + d] = (L > 0.f) ? acc / (L * pscale) : 0.f;
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
