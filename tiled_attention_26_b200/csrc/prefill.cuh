// Fused attention forward (prefill) for sm_100a.
//
// Computes O = softmax(Q K^T * scale + mask) V in one tiled pass with an online softmax, so
// the score matrix never leaves the chip ("Flash Attention on Ascend: three techniques",
// sections "tiling" and "online softmax"; "FlashAttention on Ascend NPUs", tiling section).
//
// One CTA owns 256 query rows, split into two 128-row tiles that share every K/V tile load.
// Row r of the CTA is (token tok0 + r / Gp, query head h0 + r % Gp): Gp query heads of one KV
// group are packed into the rows, so a K/V tile staged once in shared memory serves all of
// them; the head mapping is that of an explicit repeat_interleave of the KV heads ("FlashAttention
// variants: GQA, MQA, sparse attention", KV-expansion section) without ever building the copy.
//
// Warp roles (384 threads):
//   warps 0-3  softmax for Q tile 0 (thread = row = TMEM lane), warps 4-7 the same for tile 1.
//              Each reads its S row from TMEM, masks, updates the running max m and sum l,
//              writes P (bf16) back into TMEM over S, rescales O in TMEM when m grew by more
//              than 2^8, and at the end normalises O, stages it in shared memory and stores it
//              with TMA, plus the row's log-sum-exp.
//   warp 8     TMA producer: Q tiles once, then K_j, V_j into a ring of shared-memory stages;
//              both copies of tile j complete on the full barrier of K_j's stage, so the MMA
//              thread waits once per key tile.
//   warp 9     allocates TMEM and issues tcgen05.mma from one thread:
//                S_t = Q_t K_j^T (both operands in shared memory),
//                O_t += P_t V_j  (P from TMEM, V from shared memory; P arrives in two halves).
//              Order per step: PV0(j), QK0(j+1), PV1(j), QK1(j+1), so that the tensor core
//              works on one tile while the softmax warps work on the other.
//   warps 10-11 idle.
// TMEM columns: S0 [0,128), S1 [128,256), O0 [256,256+D), O1 [256+D,256+2D); P_t is the first
// 64 columns of S_t (two bf16 per column).
#pragma once

#include "sm100.cuh"

namespace fa {

struct PrefillParams {
  int B, Hq, Hkv, Sq, Skv;
  int G;       // query heads per KV head
  int Gp;      // query heads packed into the rows of one tile (power of two, divides G)
  int NP;      // G / Gp
  int n_qblocks;
  float scale_log2;  // scale * log2(e)
  int causal;
  int window;  // <= 0: none
  float* lse;  // [B, Hq, Sq] natural log, may be null
  uint64_t timeout_ns;
  // additive mask (kModeMask): fp32, element (b, h, i, j) at mask[b*mask_sb + h*mask_sh +
  // i*Skv + j]; a zero stride broadcasts
  const float* mask;
  long long mask_sb, mask_sh;
  float inv_scale;  // 1 / scale: the mask joins the raw scores as mask / scale
  int mask_vec;     // every mask row starts 16-byte aligned (Skv and both strides % 4 == 0)
  int n_global;     // kModeGlobal: tokens [0, n_global) attend to and are attended by all
};

// The key tiles one Q tile needs: [first, last], restricted (with global tokens and no global
// query in the tile) to the global tiles [0, gT) and the band [jlo, jhi).
struct TileSet {
  int first, last, jlo, jhi;
  bool allq;  // the tile holds a global query: every key tile
  template <bool kGlobal>
  __device__ __forceinline__ bool has(int j, int gT) const {
    if (j < first || j > last) return false;
    if (!kGlobal || allq) return true;
    return j < gT || (j >= jlo && j < jhi);
  }
};

// Kernel variants: an additive mask tensor, and global tokens on top of the causal / window
// rule ("FlashAttention variants: GQA, MQA, sparse attention", sliding-window section: the
// mask passed as atten_mask; global+local section).
constexpr int kModeMask = 1;
constexpr int kModeGlobal = 2;

template <int D>
struct PrefillCfg {
  static constexpr int kThreads = 384;
  static constexpr int kHalves = D / 64;          // 128-byte swizzle atoms along D
  static constexpr int kAtomBytes = 128 * 128;    // 128 rows x 128 bytes
  static constexpr int kTileBytes = 128 * D * 2;  // one 128-row bf16 tile
  static constexpr int kStages = (D == 128) ? 4 : 8;
  static constexpr int kQOff = 0;
  static constexpr int kKVOff = 2 * kTileBytes;
  static constexpr int kBarOff = kKVOff + kStages * kTileBytes;
  // barriers: q_full, kv_full[S], kv_empty[S], s_full[2], p_full[2 tiles][2 halves],
  // o_final[2], drain
  static constexpr int kBarQ = 0;
  static constexpr int kBarKVFull = 1;
  static constexpr int kBarKVEmpty = 1 + kStages;
  static constexpr int kBarSFull = 1 + 2 * kStages;
  static constexpr int kBarPFull = kBarSFull + 2;
  static constexpr int kBarOFinal = kBarPFull + 4;
  static constexpr int kBarDrain = kBarOFinal + 2;
  static constexpr int kNumBars = kBarDrain + 1;
  static constexpr int kMiscOff = kBarOff + kNumBars * 8;
  static constexpr int kSmemBytes = kMiscOff + 16 + 1024;  // + slack to align the base
  // mask variant: per softmax warp, two 16-key chunks of its 32 rows' mask (fp32), staged
  // by asynchronous copies
  static constexpr int kMaskChunk = 16;
  static constexpr int kMaskSlotBytes = 32 * kMaskChunk * 4;  // 2 KB
  static constexpr int kMaskOff = (kMiscOff + 16 + 127) / 128 * 128;
  static constexpr int kMaskBytes = 8 * 2 * kMaskSlotBytes;   // 32 KB
  static constexpr int kSmemBytesMask = kMaskOff + kMaskBytes + 1024;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr uint32_t kRegsSoftmax = 216;
  // the rest of the 384 x 168 launch registers go to the producer / MMA warpgroup
  static constexpr uint32_t kRegsOther = ((168 * 384 - 2 * 128 * kRegsSoftmax) / 128) / 8 * 8;
  static constexpr int kMinLaunchRegs =
      (2 * 128 * kRegsSoftmax + 128 * kRegsOther + kThreads - 1) / kThreads;
  __device__ static constexpr uint32_t colS(int t) { return 128u * t; }
  __device__ static constexpr uint32_t colO(int t) { return 256u + uint32_t(D) * t; }
};

// Visible keys of query token i: [vis_lo, vis_hi] (inclusive; empty when hi < lo).  Causal
// masks are aligned to the bottom-right corner; a window keeps the W nearest keys, the
// query's own position included ("FlashAttention variants: GQA, MQA, sparse attention",
// sliding-window section).
__device__ __forceinline__ int vis_lo(const PrefillParams& p, int i) {
  return p.window > 0 ? max(0, i + (p.Skv - p.Sq) - p.window + 1) : 0;
}
__device__ __forceinline__ int vis_hi(const PrefillParams& p, int i) {
  return p.causal ? min(i + (p.Skv - p.Sq), p.Skv - 1) : p.Skv - 1;
}

// Row maximum of the 128 raw scores (3-input max, 8 independent chains).
__device__ __forceinline__ float row_max128(const uint32_t (&sv)[4][32]) {
  float m[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) m[c] = -INFINITY;
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const int col = 16 * i + 2 * c;
      m[c] = fmax3(m[c], __uint_as_float(sv[col / 32][col % 32]),
                   __uint_as_float(sv[(col + 1) / 32][(col + 1) % 32]));
    }
  return fmax3(fmax3(m[0], m[1], m[2]), fmax3(m[3], m[4], m[5]), fmaxf(m[6], m[7]));
}

// p = 2^(s * sl2 - m_use) for the 64 columns of one half, written to TMEM as 32 bf16 pairs;
// returns the fp32 sum of the half through acc (two packed partial sums).
__device__ __forceinline__ void exp_half(const uint32_t (&sv)[4][32], int half, float sl2,
                                         float m_use, uint32_t taddr, uint64_t& acc0,
                                         uint64_t& acc1) {
  const uint64_t scale2 = f2(sl2, sl2), negm2 = f2(-m_use, -m_use);
  uint32_t pk[32];
#pragma unroll
  for (int k = 0; k < 32; ++k) {
    const int col = 64 * half + 2 * k;
    const uint64_t x = f2_fma(f2(__uint_as_float(sv[col / 32][col % 32]),
                                 __uint_as_float(sv[(col + 1) / 32][(col + 1) % 32])),
                              scale2, negm2);
    float x0, x1;
    f2_split(x, x0, x1);
    const float a = ex2(x0), c = ex2(x1);
    if (k & 1) acc1 = f2_add(acc1, f2(a, c)); else acc0 = f2_add(acc0, f2(a, c));
    pk[k] = pack_bf16x2(a, c);
  }
  tmem_st32(taddr + 32 * half, pk);
}

template <int D, int kMode>
__global__ void __launch_bounds__(384, 1)
    fa_prefill_kernel(const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v,
                      const __grid_constant__ CUtensorMap tm_o, const PrefillParams p) {
  using C = PrefillCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t sQ = sbase + C::kQOff;
  const uint32_t sKV = sbase + C::kKVOff;
  auto bar = [&](int idx) { return sbase + C::kBarOff + 8u * idx; };
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::kMiscOff);
  int* abort_flag = reinterpret_cast<int*>(smem + C::kMiscOff + 4);
  const WaitCtl ctl{abort_flag, p.timeout_ns};

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- work item: heaviest query blocks first: the blocks holding global queries (they see
  // every key), then the rest from the last block (the longest causal rows) down ----
  const int per_qb = p.B * p.Hkv * p.NP;
  const int order = static_cast<int>(blockIdx.x) / per_qb;
  int qb = p.n_qblocks - 1 - order;
  if constexpr ((kMode & kModeGlobal) != 0) {
    const int n_gqb = min(p.n_qblocks, (p.n_global + 256 / p.Gp - 1) / (256 / p.Gp));
    qb = order < n_gqb ? order : p.n_qblocks - 1 - (order - n_gqb);
  }
  int rem = static_cast<int>(blockIdx.x) % per_qb;
  const int b = rem / (p.Hkv * p.NP);
  rem %= p.Hkv * p.NP;
  const int g = rem / p.NP;
  const int h0 = g * p.G + (rem % p.NP) * p.Gp;
  const int tpt = 128 / p.Gp;  // tokens per tile
  const int tok0 = qb * 2 * tpt;

  // ---- key-tile range of each Q tile, and the rows that bound its masks ----
  int jlo[2], jhi[2], lo_last[2], hi_first[2];
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const int first = tok0 + t * tpt;
    const int last = min(first + tpt, p.Sq) - 1;
    jlo[t] = jhi[t] = 0;
    lo_last[t] = 0;
    hi_first[t] = -1;
    if (first < p.Sq) {
      const int lo = vis_lo(p, first), hi = vis_hi(p, last);
      lo_last[t] = vis_lo(p, last);
      hi_first[t] = vis_hi(p, first);
      if (hi >= lo && hi >= 0) {
        jlo[t] = lo / 128;
        jhi[t] = hi / 128 + 1;
      }
    }
  }
  // Key tiles each Q tile needs.  Without global tokens: the contiguous band [jlo, jhi).  With
  // G global tokens: the tiles holding keys [0, G) plus the band, or every tile when the Q
  // tile holds a global query; the tiles in between are never loaded.
  constexpr bool kGlobal = (kMode & kModeGlobal) != 0;
  constexpr bool kMask = (kMode & kModeMask) != 0;
  const int nK = (p.Skv + 127) / 128;
  const int gT = kGlobal ? min(nK, (p.n_global + 127) / 128) : 0;
  TileSet ts[2];
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const int first = tok0 + t * tpt;
    ts[t] = TileSet{jlo[t], jhi[t] - 1, jlo[t], jhi[t], false};
    if (kGlobal && first < p.Sq) {
      ts[t].allq = first < p.n_global;
      if (ts[t].allq) {
        ts[t].first = 0;
        ts[t].last = nK - 1;
      } else if (gT > 0) {
        ts[t].first = 0;
        ts[t].last = max(gT - 1, jhi[t] - 1);
      }
    }
  }
  const TileSet ts0 = ts[0], ts1 = ts[1];
  auto part = [&](int t, int j) -> bool { return (t ? ts1 : ts0).has<kGlobal>(j, gT); };
  const bool act0 = ts0.last >= ts0.first, act1 = ts1.last >= ts1.first;
  const int J0 = act0 ? (act1 ? min(ts0.first, ts1.first) : ts0.first) : (act1 ? ts1.first : 0);
  const int J1 = act0 ? (act1 ? max(ts0.last, ts1.last) : ts0.last) + 1 : (act1 ? ts1.last + 1 : 0);
  auto need = [&](int j) { return part(0, j) || part(1, j); };
  // next tile after j that some Q tile needs (J1 if none)
  auto next_need = [&](int j) {
    int x = j + 1;
    if constexpr (kGlobal)
      while (x < J1 && !need(x)) ++x;
    return x;
  };

  // ---- setup ----
  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kNumBars; ++i) {
      uint32_t count = 1;
      if (i >= C::kBarPFull && i < C::kBarPFull + 4) count = 128;
      mbar_init(bar(i), count);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 8 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    tma_prefetch_desc(&tm_o);
  }
  if (warp == 9) {
    tmem_alloc(smem_u32(tmem_holder), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  // Registers: the softmax warpgroups hold a full S row (128 fp32) per thread; the producer /
  // MMA warpgroup needs few.  2*128*216 + 128*56 = 62464 <= 384 threads * 168 at launch (the
  // host refuses to launch if the kernel was given fewer than kMinLaunchRegs per thread).
  if (warp >= 8) {
    setmaxnreg_dec<C::kRegsOther>();
  if (warp == 8) {
    // ================= TMA producer =================
    if (lane == 0) {
      int issued = 0;  // K/V copies started; slot of copy n is n % kStages
      mbar_arrive_expect_tx(bar(C::kBarQ), 2 * C::kTileBytes);
#pragma unroll
      for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int hf = 0; hf < C::kHalves; ++hf)
          tma_load_4d(sQ + t * C::kTileBytes + hf * C::kAtomBytes, &tm_q, bar(C::kBarQ), 64 * hf,
                      h0, tok0 + t * tpt, b);
      bool ok = true;
      int kt = 0;  // index of tile j among the needed tiles
      for (int j = J0; j < J1 && ok; j = next_need(j), ++kt) {
#pragma unroll
        for (int kind = 0; kind < 2; ++kind) {
          const int pos = 2 * kt + kind;
          const int s = pos % C::kStages;
          if (!mbar_wait(bar(C::kBarKVEmpty + s), ((pos / C::kStages) & 1) ^ 1, ctl)) {
            ok = false;
            break;
          }
          // K_j and V_j land on the full barrier of K_j's stage (an even stage)
          const int sf = (2 * kt) % C::kStages;
          if (kind == 0) mbar_arrive_expect_tx(bar(C::kBarKVFull + sf), 2 * C::kTileBytes);
#pragma unroll
          for (int hf = 0; hf < C::kHalves; ++hf)
            tma_load_4d(sKV + s * C::kTileBytes + hf * C::kAtomBytes, kind ? &tm_v : &tm_k,
                        bar(C::kBarKVFull + sf), 64 * hf, g, 128 * j, b);
          issued = pos + 1;
        }
      }
      // Every copy this thread started has landed before the CTA can exit (already true on
      // the normal path; after a consumer gave up this waits, bounded, for copies in flight;
      // a K_j whose V_j was never started leaves its barrier short, and that wait runs out).
      volatile int zero = 0;
      const WaitCtl drain_ctl{&zero, p.timeout_ns};
      mbar_wait(bar(C::kBarQ), 0, drain_ctl);
      for (int s = 0; s < C::kStages && s < issued; s += 2) {
        const int last = s + C::kStages * ((issued - 1 - s) / C::kStages);
        mbar_wait(bar(C::kBarKVFull + s), (last / C::kStages) & 1, drain_ctl);
      }
    }
  } else if (warp == 9) {
    // ================= MMA issuer =================
    // One thread issues both Q tiles' chains in the order PV0(j), QK0(j+1), PV1(j), QK1(j+1):
    // the tensor core finishes one tile's S while the softmax warps work on the other tile.
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 128, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, D, true);
      auto issue_qk = [&](int t, int slot) {
        const uint32_t qa = sQ + t * C::kTileBytes, kb = sKV + slot * C::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk / 4) * C::kAtomBytes + (kk % 4) * 32;
          umma_ss(tmem + C::colS(t), smem_desc_sw128(qa + off, 16, 1024),
                  smem_desc_sw128(kb + off, 16, 1024), idesc_qk, kk > 0 ? 1u : 0u);
        }
      };
      // O_t += P_t V over keys [64 * half, 64 * half + 64) of the tile
      auto issue_pv_half = [&](int t, int slot, int half, bool first) {
        const uint32_t vb = sKV + slot * C::kTileBytes;
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4) {
          const int kk = 4 * half + k4;
          umma_ts(tmem + C::colO(t), tmem + C::colS(t) + kk * 8,
                  smem_desc_sw128(vb + kk * 16 * 128, C::kAtomBytes, 1024), idesc_pv,
                  (first && kk == 0) ? 0u : 1u);
        }
      };
      // P_t arrives in two halves; the first half of PV starts while the softmax warps are
      // still computing the second.
      auto issue_pv = [&](int t, int slot, bool first, int phase) -> bool {
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          if (!mbar_wait(bar(C::kBarPFull + 2 * t + half), phase, ctl)) return false;
          tc_fence_after();
          issue_pv_half(t, slot, half, first);
        }
        return true;
      };
      // K_j and V_j in shared memory (one barrier for both, at K_j's position).  The MMAs
      // read them through the async proxy that wrote them; no tcgen05 fence is needed here.
      auto kv_wait = [&](int pos) {
        return mbar_wait(bar(C::kBarKVFull + pos % C::kStages), (pos / C::kStages) & 1, ctl);
      };
      int n[2] = {0, 0};
      bool ok = mbar_wait(bar(C::kBarQ), 0, ctl);
      if (ok && J1 > J0) {
        tc_fence_after();
        if ((ok = kv_wait(0))) {
#pragma unroll
          for (int t = 0; t < 2; ++t)
            if (part(t, J0)) {
              issue_qk(t, 0);
              tc_commit(bar(C::kBarSFull + t));
            }
          tc_commit(bar(C::kBarKVEmpty + 0));
        }
        int kt = 0;
        for (int j = J0, jn; j < J1 && ok; j = jn, ++kt) {
          jn = next_need(j);
          const int vpos = 2 * kt + 1, kpos = vpos + 1;
          const int vslot = vpos % C::kStages, kslot = kpos % C::kStages;
          const bool nxt = jn < J1;
          if (part(0, j)) {
            if (!(ok = issue_pv(0, vslot, j == ts0.first, n[0] & 1))) break;
            ++n[0];
            if (j == ts0.last) tc_commit(bar(C::kBarOFinal + 0));
          }
          if (nxt) {
            if (!(ok = kv_wait(kpos))) break;
            if (part(0, jn)) {
              issue_qk(0, kslot);
              tc_commit(bar(C::kBarSFull + 0));
            }
          }
          if (part(1, j)) {
            if (!(ok = issue_pv(1, vslot, j == ts1.first, n[1] & 1))) break;
            ++n[1];
            if (j == ts1.last) tc_commit(bar(C::kBarOFinal + 1));
          }
          tc_commit(bar(C::kBarKVEmpty + vslot));
          if (nxt) {
            if (part(1, jn)) {
              issue_qk(1, kslot);
              tc_commit(bar(C::kBarSFull + 1));
            }
            tc_commit(bar(C::kBarKVEmpty + kslot));
          }
        }
      }
      // Drain: every MMA this thread issued has completed before TMEM is released.
      tc_commit(bar(C::kBarDrain));
      volatile int zero = 0;
      const WaitCtl drain_ctl{&zero, p.timeout_ns};
      mbar_wait(bar(C::kBarDrain), 0, drain_ctl);
    }
  }  // warps 10-11 have no role
  } else {
    setmaxnreg_inc<C::kRegsSoftmax>();
    // ================= softmax + correction + epilogue =================
    const int t = warp >> 2;
    const int r = threadIdx.x & 127;
    const TileSet my_ts = t ? ts1 : ts0;
    const int t_lo_last = t ? lo_last[1] : lo_last[0];
    const int t_hi_first = t ? hi_first[1] : hi_first[0];
    const uint32_t colS = t ? C::colS(1) : C::colS(0);
    const uint32_t colO = t ? C::colO(1) : C::colO(0);
    const uint32_t trow = tmem + (static_cast<uint32_t>(32 * (warp & 3)) << 16);
    const int R = t * 128 + r;
    const int i = tok0 + R / p.Gp;
    const int hh = h0 + R % p.Gp;
    const int my_lo = vis_lo(p, i), my_hi = vis_hi(p, i);
    const int t_last_tok = min(tok0 + t * tpt + tpt, p.Sq) - 1;
    const float sl2 = p.scale_log2;
    const bool mvec = p.mask_vec != 0;  // rows start 16-byte aligned: staged vector copies
    // Mask staging (kMask, mvec): this warp's 32 rows, 16 keys at a time, copied with 16-byte
    // cp.async (lane: row (lane >> 2) + 8 it, bytes 16 (lane & 3)) into two 2 KB slots; a row's
    // 16-byte pieces sit at (row, piece ^ ((row >> 1) & 3)) so that the row-per-lane reads
    // spread over all banks.  Chunk number mseq runs across tiles; chunk 0 of the next tile is
    // requested while this tile's last chunk is read.
    int mseq = 0;
    // the first of the four rows this lane copies (the others follow 8 rows apart)
    const int crow0 = t * 128 + 32 * (warp & 3) + (lane >> 2);
    uint8_t* const mbase = smem + C::kMaskOff + warp * 2 * C::kMaskSlotBytes;
    auto mslot = [&](int slot) -> const uint8_t* { return mbase + slot * C::kMaskSlotBytes; };
    // copy chunk k (keys 16k.. of key tile jt) into slot `slot`
    auto mask_issue = [&](int jt, int k, int slot) {
#pragma unroll
      for (int it = 0; it < 4; ++it) {
        const int row = (lane >> 2) + 8 * it, pc = lane & 3;
        const int key = 128 * jt + C::kMaskChunk * k + 4 * pc;
        const int Rr = crow0 + 8 * it;
        const int ir = tok0 + Rr / p.Gp, hr = h0 + Rr % p.Gp;
        const bool ok = ir < p.Sq && key < p.Skv;
        const float* src = ok ? p.mask + b * p.mask_sb + hr * p.mask_sh +
                                    static_cast<long long>(ir) * p.Skv + key
                              : p.mask;
        const uint32_t dst = smem_u32(mbase + slot * C::kMaskSlotBytes + row * 64 +
                                      16 * (pc ^ ((row >> 1) & 3)));
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
                     "r"(ok ? 16 : 0)
                     : "memory");
      }
      asm volatile("cp.async.commit_group;" ::: "memory");
    };
    // next needed key tile of this Q tile after jt (or -1)
    auto next_tile = [&](int jt) -> int {
      for (int x = jt + 1; x <= my_ts.last; ++x)
        if (my_ts.has<kGlobal>(x, gT)) return x;
      return -1;
    };
    // before reading chunk k of tile jt (chunk number mseq): request the following chunk, then
    // wait until this one has landed
    auto mask_stage = [&](int jt, int k) {
      bool more = true;
      if (k + 1 < 128 / C::kMaskChunk) {
        mask_issue(jt, k + 1, (mseq + 1) & 1);
      } else {
        const int jn = next_tile(jt);
        if (jn >= 0) mask_issue(jn, 0, (mseq + 1) & 1); else more = false;
      }
      if (more) asm volatile("cp.async.wait_group 1;" ::: "memory");
      else asm volatile("cp.async.wait_group 0;" ::: "memory");
      __syncwarp();
    };
    if constexpr (kMask)
      if (mvec && my_ts.last >= my_ts.first) mask_issue(my_ts.first, 0, 0);
    float m = -INFINITY, l = 0.f;
    int n = 0;
    for (int j = my_ts.first; j <= my_ts.last; ++j) {
      if constexpr (kGlobal)
        if (!my_ts.has<kGlobal>(j, gT)) continue;
      bool ok = mbar_wait(bar(C::kBarSFull + t), n & 1, ctl);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      uint32_t sv[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(trow + colS + 32 * c, sv[c]);
      tmem_wait_ld();
      if constexpr (kMask) {
        // scores += mask / scale (the exponent then carries scale * s + mask, in log2 units)
        if (mvec) {
          // the mask chunks were staged in shared memory by coalesced asynchronous copies
#pragma unroll
          for (int k = 0; k < 128 / C::kMaskChunk; ++k) {
            mask_stage(j, k);  // issues the next chunk, waits for this one
#pragma unroll
            for (int pc = 0; pc < 4; ++pc) {
              const float4 x = *reinterpret_cast<const float4*>(
                  mslot(mseq & 1) + (r & 31) * 64 + 16 * (pc ^ (((r & 31) >> 1) & 3)));
              const float mv[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int col = C::kMaskChunk * k + 4 * pc + e;
                sv[col / 32][col % 32] = __float_as_uint(
                    fmaf(mv[e], p.inv_scale, __uint_as_float(sv[col / 32][col % 32])));
              }
            }
            __syncwarp();  // every lane has read the slot before it is refilled
            ++mseq;
          }
        } else if (i < p.Sq) {
          // rows not 16-byte aligned: this row's values, one at a time
          const float* mrow =
              p.mask + b * p.mask_sb + hh * p.mask_sh + static_cast<long long>(i) * p.Skv;
#pragma unroll
          for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int q4 = 0; q4 < 8; ++q4) {
              const int key = 128 * j + 32 * c + 4 * q4;
              float mv[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
              for (int e = 0; e < 4; ++e)
                if (key + e < p.Skv) mv[e] = __ldg(mrow + key + e);
#pragma unroll
              for (int e = 0; e < 4; ++e)
                sv[c][4 * q4 + e] = __float_as_uint(
                    fmaf(mv[e], p.inv_scale, __uint_as_float(sv[c][4 * q4 + e])));
            }
        }
      }
      bool need_mask = (128 * j < t_lo_last) || (128 * j + 127 > t_hi_first);
      if constexpr (kGlobal) {
        const bool full = (128 * j + 127 < p.Skv) &&
                          (t_last_tok < p.n_global || 128 * j + 127 < p.n_global || !need_mask);
        need_mask = !full;
      }
      if (need_mask) {
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int k = 0; k < 32; ++k) {
            const int key = 128 * j + 32 * c + k;
            bool vis = key >= my_lo && key <= my_hi;
            if constexpr (kGlobal)
              vis = vis || (key < p.Skv && (key < p.n_global || i < p.n_global));
            if (!vis) sv[c][k] = __float_as_uint(-INFINITY);
          }
      }
      const float m_tile = row_max128(sv) * sl2;
      const float m_new = fmaxf(m, m_tile);
      float alpha = 1.f;
      bool resc = false;
      if (n == 0) {
        m = m_new;
      } else if (m_new > m + 8.f) {
        resc = true;
        alpha = ex2(m - m_new);
        m = m_new;
      }
      // Lazy correction: O (accumulated up to the previous tile, complete since S of this tile
      // is) is rescaled only when the running max grew by more than 2^8; otherwise the stale max
      // stays the reference and p may reach 2^8, which fp32 O and l absorb exactly.
      if (__any_sync(0xffffffffu, resc)) {
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t ov[32];
          tmem_ld32(trow + colO + 32 * c, ov);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; ++k) ov[k] = __float_as_uint(__uint_as_float(ov[k]) * alpha);
          tmem_st32(trow + colO + 32 * c, ov);
        }
      }
      const float m_use = (m == -INFINITY) ? 0.f : m;
      // p = 2^(s * scale * log2(e) - m) as bf16 pairs over the S columns, one half at a time;
      // each half is released to the MMA warp as soon as it is in TMEM.
      uint64_t acc0 = f2(0.f, 0.f), acc1 = f2(0.f, 0.f);
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        // (the two identical calls keep the register allocation of the plain path spill-free)
        if (need_mask || kMask)
          exp_half(sv, half, sl2, m_use, trow + colS, acc0, acc1);
        else
          exp_half(sv, half, sl2, m_use, trow + colS, acc0, acc1);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar(C::kBarPFull + 2 * t + half));
      }
      float a0, a1, a2, a3;
      f2_split(acc0, a0, a1);
      f2_split(acc1, a2, a3);
      l = l * alpha + ((a0 + a1) + (a2 + a3));
      ++n;
    }

    // mask copies still in flight (after an abandoned wait) land before the CTA moves on
    if constexpr (kMask) asm volatile("cp.async.wait_all;" ::: "memory");

    // ---- epilogue: O / l -> bf16 -> shared memory (swizzled like the O tensor map) -> TMA ----
    bool have_o = false;
    if (n > 0) {
      bool ok = mbar_wait(bar(C::kBarOFinal + t), 0, ctl);
      have_o = __all_sync(0xffffffffu, ok);
      tc_fence_after();
    } else {
      // no product ran for this tile: the Q copy into its staging buffer may still be landing
      mbar_wait(bar(C::kBarQ), 0, ctl);
    }
    const float inv_l = (l > 0.f) ? 1.f / l : 0.f;
    const uint32_t stage = sQ + t * C::kTileBytes;  // Q tile t is no longer read
    uint8_t* stage_ptr = smem + C::kQOff + t * C::kTileBytes;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      uint32_t ov[32];
      if (have_o) {
        tmem_ld32(trow + colO + 32 * c, ov);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int k = 0; k < 32; ++k) ov[k] = 0u;
      }
      const int hf = c >> 1;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint4 w;
        w.x = pack_bf16x2(__uint_as_float(ov[8 * q + 0]) * inv_l, __uint_as_float(ov[8 * q + 1]) * inv_l);
        w.y = pack_bf16x2(__uint_as_float(ov[8 * q + 2]) * inv_l, __uint_as_float(ov[8 * q + 3]) * inv_l);
        w.z = pack_bf16x2(__uint_as_float(ov[8 * q + 4]) * inv_l, __uint_as_float(ov[8 * q + 5]) * inv_l);
        w.w = pack_bf16x2(__uint_as_float(ov[8 * q + 6]) * inv_l, __uint_as_float(ov[8 * q + 7]) * inv_l);
        const int chunk = ((c & 1) * 4 + q) ^ (r & 7);
        *reinterpret_cast<uint4*>(stage_ptr + hf * C::kAtomBytes + r * 128 + chunk * 16) = w;
      }
    }
    fence_proxy_async_smem();
    named_bar_sync(1 + t, 128);
    if (r == 0 && tok0 + t * tpt < p.Sq) {
#pragma unroll
      for (int hf = 0; hf < C::kHalves; ++hf)
        tma_store_4d(&tm_o, stage + hf * C::kAtomBytes, 64 * hf, h0, tok0 + t * tpt, b);
      tma_store_commit();
      tma_store_wait_read_all();
    }
    if (p.lse != nullptr && i < p.Sq) {
      const float lse = (l > 0.f) ? (m + __log2f(l)) * 0.69314718055994531f : -INFINITY;
      p.lse[(static_cast<size_t>(b) * p.Hq + hh) * p.Sq + i] = lse;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

}  // namespace fa
