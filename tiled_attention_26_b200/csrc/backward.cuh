// Attention backward pass for sm_100a.
//
// The forward pass keeps only O and the row log-sum-exp; the backward pass recomputes the
// probabilities tile by tile instead of storing them ("FlashAttention on Ascend NPUs",
// recomputation section).  With L the row log-sum-exp and D_i = dO_i . O_i:
//   P_ij = exp(scale q_i.k_j - L_i),  dP_ij = dO_i . v_j,  dS_ij = P_ij (dP_ij - D_i)
//   dV_j = sum_i P_ij dO_i,  dK_j = scale sum_i dS_ij q_i,  dQ_i = scale sum_j dS_ij k_j
// Three kernels, none with atomics:
//   fa_bwd_prep_kernel   -D_i and -L_i * log2(e) per (b, h, i) into a padded workspace
//                        (padding rows get L = +inf, D = 0: they contribute nothing);
//   fa_bwd_dkdv_kernel   one CTA per (b, KV head, 128-key tile): S^T = K Q^T and
//                        dP^T = V dO^T per (query head of the group, 128-query tile), then
//                        dV += P^T dO and dK += dS^T Q with P and dS in TMEM (GQA heads summed
//                        in TMEM), one bf16 store of dK and dV at the end;
//   fa_bwd_dq_kernel     one CTA per 128-row Q tile (query heads packed into rows as in the
//                        forward pass): S = Q K^T and dP = dO V^T per key tile, then
//                        dQ += dS K with dS in TMEM.
// Warp roles (320 threads): warps 0-7 elementwise (thread = row = TMEM lane of its quadrant;
// warps w and w + 4 share a quadrant and take one half of the columns each), warp 8 TMA
// producer, warp 9 TMEM allocation + tcgen05.mma issue from one thread.
#pragma once

#include "prefill.cuh"
#include "sm100.cuh"

namespace fa {

struct BwdParams {
  int B, Hq, Hkv, Sq, Skv;
  int G, Gp, NP;
  int Sq_pad;          // rows of the per-(b, h) workspace vectors (multiple of 128)
  int n_tiles;         // dQ: 128-row Q tiles per (b, KV head, head pack); dK/dV: key tiles
  float scale;         // softmax scale
  float scale_log2;    // scale * log2(e)
  int causal, window;
  const uint16_t* o;     // bf16 [B, Sq, Hq, D]
  const uint16_t* dout;  // bf16 [B, Sq, Hq, D]
  const float* lse;      // natural log [B, Hq, Sq]
  float* lse2;           // workspace [B * Hq, Sq_pad]: -L * log2(e)
  float* delta;          // workspace [B * Hq, Sq_pad]: -D
  uint64_t timeout_ns;
};

template <int D>
struct BwdCfg {
  static constexpr int kThreads = 320;
  static constexpr int kHalves = D / 64;
  static constexpr int kAtomBytes = 128 * 128;
  static constexpr int kTileBytes = 128 * D * 2;
  static constexpr uint32_t kTmemCols = 512;
  // dQ kernel: Q and dO tiles, then a K/V ring
  static constexpr int kQStages = (D == 128) ? 4 : 8;
  static constexpr int kQOff = 0;
  static constexpr int kDOOff = kTileBytes;
  static constexpr int kQKVOff = 2 * kTileBytes;
  static constexpr int kQBarOff = kQKVOff + kQStages * kTileBytes;
  // barriers: in_full, kv_full[S], kv_empty[S], sdp_full, sdp_free, ds_ready, dq_done,
  // o_final, drain
  static constexpr int kQNumBars = 7 + 2 * kQStages;
  static constexpr int kQMiscOff = kQBarOff + 8 * kQNumBars;
  static constexpr int kQSmemBytes = kQMiscOff + 16 + 1024;
  // dK/dV kernel: K and V tiles, then a ring of (Q, dO, L, D) units
  static constexpr int kUStages = (D == 128) ? 2 : 4;
  static constexpr int kUnitBytes = 2 * kTileBytes + 2 * 128 * 4;
  static constexpr int kKOff = 0;
  static constexpr int kVOff = kTileBytes;
  static constexpr int kUOff = 2 * kTileBytes;
  static constexpr int kUBarOff = kUOff + kUStages * kUnitBytes;
  // barriers: kv_full, u_full[S] (Q and the vectors), u_empty[S], s_full, dp_full, p_ready,
  // ds_ready, o_final, drain, u_do[S] (dO)
  static constexpr int kUNumBars = 7 + 3 * kUStages;
  static constexpr int kUMiscOff = kUBarOff + 8 * kUNumBars;
  static constexpr int kUSmemBytes = kUMiscOff + 16 + 1024;
};

// ---------------------------------------------------------------------------------------
// -D_i = -dO_i . O_i and -L_i * log2(e) per (b, h, i) row, D / 8 lanes per row (stored negated
// so the kernels add them); padding rows past Sq get L = +inf and D = 0.  Rows with L = -inf (no
// visible key) also get +inf: their P is 0.
// ---------------------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) fa_bwd_prep_kernel(const BwdParams p) {
  // D / 8 lanes per row, one 16-byte load of O and of dO each (8 bf16); 256 / D rows per warp
  constexpr int kLanesPerRow = D / 8;
  constexpr int kRowsPerWarp = 32 / kLanesPerRow;
  const int lane = threadIdx.x & 31;
  const int sub = lane % kLanesPerRow;
  const long long row =
      (static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5)) * kRowsPerWarp +
      lane / kLanesPerRow;
  const long long rows = static_cast<long long>(p.B) * p.Hq * p.Sq_pad;
  const bool valid = row < rows;  // no early exit: the row's lanes reduce with shuffles
  const int i = valid ? static_cast<int>(row % p.Sq_pad) : 0;
  const long long bh = valid ? row / p.Sq_pad : 0;
  const int h = static_cast<int>(bh % p.Hq), b = static_cast<int>(bh / p.Hq);
  float acc = 0.f;
  if (valid && i < p.Sq) {
    const size_t base = ((static_cast<size_t>(b) * p.Sq + i) * p.Hq + h) * D + 8 * sub;
    const uint4 o4 = __ldg(reinterpret_cast<const uint4*>(p.o + base));
    const uint4 d4 = __ldg(reinterpret_cast<const uint4*>(p.dout + base));
    const uint32_t ow[4] = {o4.x, o4.y, o4.z, o4.w}, dw[4] = {d4.x, d4.y, d4.z, d4.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      acc = fmaf(__uint_as_float(ow[e] << 16), __uint_as_float(dw[e] << 16), acc);
      acc = fmaf(__uint_as_float(ow[e] & 0xFFFF0000u), __uint_as_float(dw[e] & 0xFFFF0000u), acc);
    }
  }
#pragma unroll
  for (int s = kLanesPerRow / 2; s > 0; s >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, s);
  if (valid && sub == 0) {
    float l2 = INFINITY;
    if (i < p.Sq) {
      const float l = p.lse[(static_cast<size_t>(b) * p.Hq + h) * p.Sq + i];
      l2 = (l == -INFINITY) ? INFINITY : l * 1.4426950408889634f;
    }
    p.lse2[row] = -l2;
    p.delta[row] = (i < p.Sq) ? -acc : 0.f;
  }
}

// Query token i sees key k (bottom-right causal alignment, window of W keys).
__device__ __forceinline__ bool bwd_visible(const BwdParams& p, int i, int k) {
  const int ip = i + (p.Skv - p.Sq);
  if (i >= p.Sq || k >= p.Skv) return false;
  if (p.causal && k > ip) return false;
  if (p.window > 0 && k <= ip - p.window) return false;
  return true;
}

// ---------------------------------------------------------------------------------------
// dK, dV: one CTA per (b, KV head g, key tile j).
// ---------------------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(320, 1)
    fa_bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v,
                       const __grid_constant__ CUtensorMap tm_do,
                       const __grid_constant__ CUtensorMap tm_vec,
                       const __grid_constant__ CUtensorMap tm_dk,
                       const __grid_constant__ CUtensorMap tm_dv, const BwdParams p) {
  using C = BwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  auto bar = [&](int idx) { return sb + C::kUBarOff + 8u * idx; };
  constexpr int kBarKV = 0, kBarUFull = 1, kBarUEmpty = 1 + C::kUStages;
  constexpr int kBarS = 1 + 2 * C::kUStages, kBarDP = kBarS + 1, kBarP = kBarS + 2,
                kBarDS = kBarS + 3, kBarO = kBarS + 4, kBarDrain = kBarS + 5,
                kBarUDo = kBarS + 6;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::kUMiscOff);
  int* abort_flag = reinterpret_cast<int*>(smem + C::kUMiscOff + 4);
  const WaitCtl ctl{abort_flag, p.timeout_ns};
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // heaviest key tiles (the first ones under a causal mask) first, every (b, KV head) of a
  // key tile before the next key tile
  const int j = static_cast<int>(blockIdx.x) / (p.B * p.Hkv);
  const int bg = static_cast<int>(blockIdx.x) % (p.B * p.Hkv);
  const int g = bg % p.Hkv, b = bg / p.Hkv;
  const int k0 = 128 * j;
  // query tiles whose rows see some key of [k0, k0 + 127]
  const int off = p.Skv - p.Sq;
  int i_lo = 0, i_hi = p.Sq - 1;
  if (p.causal) i_lo = max(0, k0 - off);
  if (p.window > 0) i_hi = min(p.Sq - 1, k0 + 127 + p.window - 1 - off);
  const int qt_lo = i_lo / 128, qt_hi = (i_hi >= i_lo) ? i_hi / 128 : qt_lo - 1;
  const int n_qt = max(0, qt_hi - qt_lo + 1);
  const int n_units = n_qt * p.G;  // unit u: head g*G + u / n_qt, query tile qt_lo + u % n_qt

  if (threadIdx.x == 0) {
    for (int x = 0; x < C::kUNumBars; ++x)
      mbar_init(bar(x), (x == kBarP || x == kBarDS) ? 256 : 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(smem_u32(tmem_holder), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  constexpr uint32_t colS = 0, colDP = 128, colDV = 256, colDK = 256 + D;

  if (warp == 8) {
    // ============ producer ============
    if (lane == 0 && n_units > 0) {
      // (with no unit the epilogue writes zeros into these tiles: nothing may land there)
      mbar_arrive_expect_tx(bar(kBarKV), 2 * C::kTileBytes);
#pragma unroll
      for (int hf = 0; hf < C::kHalves; ++hf) {
        tma_load_4d(sb + C::kKOff + hf * C::kAtomBytes, &tm_k, bar(kBarKV), 64 * hf, g, k0, b);
        tma_load_4d(sb + C::kVOff + hf * C::kAtomBytes, &tm_v, bar(kBarKV), 64 * hf, g, k0, b);
      }
      int issued = 0;
      for (int u = 0; u < n_units; ++u) {
        const int s = u % C::kUStages;
        if (u >= C::kUStages &&
            !mbar_wait(bar(kBarUEmpty + s), ((u / C::kUStages) - 1) & 1, ctl))
          break;
        const int h = g * p.G + u / n_qt, i0 = 128 * (qt_lo + u % n_qt);
        const uint32_t base = sb + C::kUOff + s * C::kUnitBytes;
        // Q and the vectors first (S^T needs them), dO on a barrier of its own (dP^T)
        mbar_arrive_expect_tx(bar(kBarUFull + s), C::kTileBytes + 1024);
#pragma unroll
        for (int hf = 0; hf < C::kHalves; ++hf)
          tma_load_4d(base + hf * C::kAtomBytes, &tm_q, bar(kBarUFull + s), 64 * hf, h, i0, b);
        // L and D vectors: rows (b*Hq + h) of the two [B*Hq, Sq_pad] workspace arrays, which
        // the vector map sees as one (Sq_pad, B*Hq, 2) tensor
        const uint32_t vb = base + 2 * C::kTileBytes;
        tma_load_3d(vb, &tm_vec, bar(kBarUFull + s), i0, b * p.Hq + h, 0);
        tma_load_3d(vb + 512, &tm_vec, bar(kBarUFull + s), i0, b * p.Hq + h, 1);
        mbar_arrive_expect_tx(bar(kBarUDo + s), C::kTileBytes);
#pragma unroll
        for (int hf = 0; hf < C::kHalves; ++hf)
          tma_load_4d(base + C::kTileBytes + hf * C::kAtomBytes, &tm_do, bar(kBarUDo + s),
                      64 * hf, h, i0, b);
        issued = u + 1;
      }
      volatile int zero = 0;
      const WaitCtl drain_ctl{&zero, p.timeout_ns};
      mbar_wait(bar(kBarKV), 0, drain_ctl);
      for (int s = 0; s < C::kUStages && s < issued; ++s) {
        const int last = s + C::kUStages * ((issued - 1 - s) / C::kUStages);
        mbar_wait(bar(kBarUFull + s), (last / C::kUStages) & 1, drain_ctl);
        mbar_wait(bar(kBarUDo + s), (last / C::kUStages) & 1, drain_ctl);
      }
    }
  } else if (warp == 9) {
    // ============ MMA issuer ============
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, false);
      constexpr uint32_t idesc_acc = idesc_bf16_f32(128, D, true);
      // D[tmem] = A_tile (K-major rows) . B_tile^T, K = D
      auto mma_rows = [&](uint32_t d, uint32_t a, uint32_t bt) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t o2 = (kk / 4) * C::kAtomBytes + (kk % 4) * 32;
          umma_ss(tmem + d, smem_desc_sw128(a + o2, 16, 1024), smem_desc_sw128(bt + o2, 16, 1024),
                  idesc_s, kk > 0 ? 1u : 0u);
        }
      };
      // D[tmem] (+)= A[tmem bf16, 128 x 128] . B_tile (MN-major, K = the tile's 128 rows);
      // A's queries 0-63 sit in columns [a_col, a_col + 32), queries 64-127 in
      // [a_col + 64, a_col + 96)
      auto mma_acc = [&](uint32_t d, uint32_t a_col, uint32_t bt, bool first) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_ts(tmem + d, tmem + a_col + 64 * (kk / 4) + 8 * (kk % 4),
                  smem_desc_sw128(bt + kk * 16 * 128, C::kAtomBytes, 1024), idesc_acc,
                  (first && kk == 0) ? 0u : 1u);
      };
      // Order: S(0) dP(0) | dV(u) S(u+1) | dK(u) dP(u+1) | ...: the tensor core works on the
      // next unit's products while the elementwise warps turn S into P and dP into dS.
      auto unit_tiles = [&](int u, uint32_t& qt, uint32_t& dot) {
        qt = sb + C::kUOff + (u % C::kUStages) * C::kUnitBytes;
        dot = qt + C::kTileBytes;
      };
      // (waits on copies into shared memory need no tcgen05 fence: the MMAs read through the
      // async proxy that wrote them; waits on TMEM written by other warps do)
      bool ok = n_units > 0 && mbar_wait(bar(kBarKV), 0, ctl);
      if (ok && (ok = mbar_wait(bar(kBarUFull), 0, ctl))) {
        uint32_t qt, dot;
        unit_tiles(0, qt, dot);
        mma_rows(colS, sb + C::kKOff, qt);    // S^T = K Q^T
        tc_commit(bar(kBarS));
        if ((ok = mbar_wait(bar(kBarUDo), 0, ctl))) {
          mma_rows(colDP, sb + C::kVOff, dot);  // dP^T = V dO^T
          tc_commit(bar(kBarDP));
        }
      }
      for (int u = 0; u < n_units && ok; ++u) {
        uint32_t qt, dot, qn = 0, don = 0;
        unit_tiles(u, qt, dot);
        const bool nxt = u + 1 < n_units;
        if (!(ok = mbar_wait(bar(kBarP), u & 1, ctl))) break;
        tc_fence_after();
        mma_acc(colDV, colS, dot, u == 0);    // dV += P^T dO
        if (nxt) {
          if (!(ok = mbar_wait(bar(kBarUFull + (u + 1) % C::kUStages), ((u + 1) / C::kUStages) & 1, ctl)))
            break;
          unit_tiles(u + 1, qn, don);
          mma_rows(colS, sb + C::kKOff, qn);  // S^T of the next unit (after dV read P)
          tc_commit(bar(kBarS));
        }
        if (!(ok = mbar_wait(bar(kBarDS), u & 1, ctl))) break;
        tc_fence_after();
        mma_acc(colDK, colDP, qt, u == 0);    // dK += dS^T Q
        tc_commit(bar(kBarUEmpty + u % C::kUStages));
        if (nxt) {
          if (!(ok = mbar_wait(bar(kBarUDo + (u + 1) % C::kUStages), ((u + 1) / C::kUStages) & 1, ctl)))
            break;
          mma_rows(colDP, sb + C::kVOff, don);  // dP^T of the next unit (after dK read dS)
          tc_commit(bar(kBarDP));
        }
      }
      tc_commit(bar(kBarO));
      tc_commit(bar(kBarDrain));
      volatile int zero = 0;
      const WaitCtl drain_ctl{&zero, p.timeout_ns};
      mbar_wait(bar(kBarDrain), 0, drain_ctl);
    }
  } else {
    // ============ elementwise: thread = key row; this warp's half of the query columns ====
    const int wq = warp & 3, ch = warp >> 2;
    const int r = 32 * wq + lane;
    const int key = k0 + r;
    const uint32_t trow = tmem + (static_cast<uint32_t>(32 * wq) << 16);
    const uint64_t sl2 = f2(p.scale_log2, p.scale_log2);
    for (int u = 0; u < n_units; ++u) {
      const int s = u % C::kUStages;
      const int i0 = 128 * (qt_lo + u % n_qt);
      // -L log2(e) and -D of the unit's 128 queries (broadcast reads, four at a time)
      const float4* vl = reinterpret_cast<const float4*>(smem + C::kUOff + s * C::kUnitBytes +
                                                         2 * C::kTileBytes) + 16 * ch;
      const float4* vd = vl + 32;
      // every (query, key) of the tile visible?  (then no per-element test)
      const bool full = bwd_visible(p, i0, k0 + 127) && bwd_visible(p, i0 + 127, k0);
      // ---- P = 2^(S^T scale log2 e - L) over this warp's 64 query columns, kept as bf16 ----
      bool ok = mbar_wait(bar(kBarS), u & 1, ctl);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      uint32_t pk[32];
      {
        uint32_t sv[64];
        tmem_ld32(trow + colS + 64 * ch, *reinterpret_cast<uint32_t(*)[32]>(sv));
        tmem_ld32(trow + colS + 64 * ch + 32, *reinterpret_cast<uint32_t(*)[32]>(sv + 32));
        tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          const float4 nl = vl[q];
          float x0, x1, x2, x3;
          f2_split(f2_fma(f2(__uint_as_float(sv[4 * q]), __uint_as_float(sv[4 * q + 1])), sl2,
                          f2(nl.x, nl.y)), x0, x1);
          f2_split(f2_fma(f2(__uint_as_float(sv[4 * q + 2]), __uint_as_float(sv[4 * q + 3])), sl2,
                          f2(nl.z, nl.w)), x2, x3);
          float e[4] = {ex2(x0), ex2(x1), ex2(x2), ex2(x3)};
          if (!full) {
#pragma unroll
            for (int t = 0; t < 4; ++t)
              if (!bwd_visible(p, i0 + 64 * ch + 4 * q + t, key)) e[t] = 0.f;
          }
          pk[2 * q] = pack_bf16x2(e[0], e[1]);
          pk[2 * q + 1] = pack_bf16x2(e[2], e[3]);
        }
      }
      // each warp writes its 64 queries' P (32 bf16 pairs) over the first half of the S^T
      // columns it read itself, so the two warps of a quadrant never touch each other's input
      tmem_st32(trow + colS + 64 * ch, pk);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(kBarP));
      // ---- dS = P (dP^T - D) ----
      ok = mbar_wait(bar(kBarDP), u & 1, ctl);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      {
        uint32_t dv[64];
        tmem_ld32(trow + colDP + 64 * ch, *reinterpret_cast<uint32_t(*)[32]>(dv));
        tmem_ld32(trow + colDP + 64 * ch + 32, *reinterpret_cast<uint32_t(*)[32]>(dv + 32));
        tmem_wait_ld();
        uint32_t ds[32];
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          const float4 nd = vd[q];
          const uint64_t p01 = f2(__uint_as_float(pk[2 * q] << 16),
                                  __uint_as_float(pk[2 * q] & 0xFFFF0000u));
          const uint64_t p23 = f2(__uint_as_float(pk[2 * q + 1] << 16),
                                  __uint_as_float(pk[2 * q + 1] & 0xFFFF0000u));
          float d0, d1, d2, d3;
          f2_split(f2_mul(p01, f2_add(f2(__uint_as_float(dv[4 * q]), __uint_as_float(dv[4 * q + 1])),
                                      f2(nd.x, nd.y))), d0, d1);
          f2_split(f2_mul(p23, f2_add(f2(__uint_as_float(dv[4 * q + 2]), __uint_as_float(dv[4 * q + 3])),
                                      f2(nd.z, nd.w))), d2, d3);
          ds[2 * q] = pack_bf16x2(d0, d1);
          ds[2 * q + 1] = pack_bf16x2(d2, d3);
        }
        tmem_st32(trow + colDP + 64 * ch, ds);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(kBarDS));
    }
    // ---- epilogue: warps 0-3 write dV, warps 4-7 scale * dK: bf16 -> swizzled smem (the
    // V / K tiles) -> TMA ----
    bool have = false;
    if (n_units > 0) {
      bool ok = mbar_wait(bar(kBarO), 0, ctl);
      have = __all_sync(0xffffffffu, ok);
      tc_fence_after();
    }
    {
      const uint32_t col = ch ? colDK : colDV;
      const float mul = ch ? p.scale : 1.f;
      uint8_t* stage = smem + (ch ? C::kKOff : C::kVOff);
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t ov[32];
        if (have) {
          tmem_ld32(trow + col + 32 * c, ov);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int x = 0; x < 32; ++x) ov[x] = 0u;
        }
        const int hf = c >> 1;
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          uint4 w;
          w.x = pack_bf16x2(__uint_as_float(ov[8 * q4 + 0]) * mul, __uint_as_float(ov[8 * q4 + 1]) * mul);
          w.y = pack_bf16x2(__uint_as_float(ov[8 * q4 + 2]) * mul, __uint_as_float(ov[8 * q4 + 3]) * mul);
          w.z = pack_bf16x2(__uint_as_float(ov[8 * q4 + 4]) * mul, __uint_as_float(ov[8 * q4 + 5]) * mul);
          w.w = pack_bf16x2(__uint_as_float(ov[8 * q4 + 6]) * mul, __uint_as_float(ov[8 * q4 + 7]) * mul);
          const int chunk = ((c & 1) * 4 + q4) ^ (r & 7);
          *reinterpret_cast<uint4*>(stage + hf * C::kAtomBytes + r * 128 + chunk * 16) = w;
        }
      }
    }
    fence_proxy_async_smem();
    named_bar_sync(1, 256);
    if (threadIdx.x == 0) {
#pragma unroll
      for (int hf = 0; hf < C::kHalves; ++hf) {
        tma_store_4d(&tm_dv, sb + C::kVOff + hf * C::kAtomBytes, 64 * hf, g, k0, b);
        tma_store_4d(&tm_dk, sb + C::kKOff + hf * C::kAtomBytes, 64 * hf, g, k0, b);
      }
      tma_store_commit();
      tma_store_wait_read_all();
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

// ---------------------------------------------------------------------------------------
// dQ: one CTA per 128-row Q tile; row r = (token t0 + r / Gp, head h0 + r % Gp).
// ---------------------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(320, 1)
    fa_bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q,
                     const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v,
                     const __grid_constant__ CUtensorMap tm_do,
                     const __grid_constant__ CUtensorMap tm_dq, const BwdParams p) {
  using C = BwdCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  auto bar = [&](int idx) { return sb + C::kQBarOff + 8u * idx; };
  constexpr int kBarIn = 0, kBarKVFull = 1, kBarKVEmpty = 1 + C::kQStages;
  constexpr int kBarSDP = 1 + 2 * C::kQStages, kBarFree = kBarSDP + 1, kBarDS = kBarSDP + 2,
                kBarDQ = kBarSDP + 3, kBarO = kBarSDP + 4, kBarDrain = kBarSDP + 5;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + C::kQMiscOff);
  int* abort_flag = reinterpret_cast<int*>(smem + C::kQMiscOff + 4);
  const WaitCtl ctl{abort_flag, p.timeout_ns};
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // heaviest (last) query tiles first
  const int per_tile = p.B * p.Hkv * p.NP;
  const int qt = p.n_tiles - 1 - static_cast<int>(blockIdx.x) / per_tile;
  int rem = static_cast<int>(blockIdx.x) % per_tile;
  const int b = rem / (p.Hkv * p.NP);
  rem %= p.Hkv * p.NP;
  const int g = rem / p.NP;
  const int h0 = g * p.G + (rem % p.NP) * p.Gp;
  const int tpt = 128 / p.Gp;
  const int tok0 = qt * tpt;
  // key tiles: the band of the tile's first and last tokens
  const int first = tok0, last = min(tok0 + tpt, p.Sq) - 1;
  const int off = p.Skv - p.Sq;
  int jlo = 0, jhi = 0;
  {
    const int lo = p.window > 0 ? max(0, first + off - p.window + 1) : 0;
    const int hi = p.causal ? min(last + off, p.Skv - 1) : p.Skv - 1;
    if (hi >= lo && hi >= 0) {
      jlo = lo / 128;
      jhi = hi / 128 + 1;
    }
  }
  const int n_kt = jhi - jlo;

  if (threadIdx.x == 0) {
    for (int x = 0; x < C::kQNumBars; ++x)
      mbar_init(bar(x), (x == kBarFree || x == kBarDS) ? 256 : 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(smem_u32(tmem_holder), C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  constexpr uint32_t colS = 0, colDP = 128, colDQ = 256, colDS = 384;

  if (warp == 8) {
    // ============ producer ============
    if (lane == 0 && n_kt > 0) {
      // (with no key tile the epilogue writes zeros into the Q tile: nothing may land there)
      mbar_arrive_expect_tx(bar(kBarIn), 2 * C::kTileBytes);
#pragma unroll
      for (int hf = 0; hf < C::kHalves; ++hf) {
        tma_load_4d(sb + C::kQOff + hf * C::kAtomBytes, &tm_q, bar(kBarIn), 64 * hf, h0, tok0, b);
        tma_load_4d(sb + C::kDOOff + hf * C::kAtomBytes, &tm_do, bar(kBarIn), 64 * hf, h0, tok0, b);
      }
      int issued = 0;
      bool ok = true;
      for (int t = 0; t < n_kt && ok; ++t) {
#pragma unroll
        for (int kind = 0; kind < 2; ++kind) {
          const int pos = 2 * t + kind;
          const int s = pos % C::kQStages;
          if (!mbar_wait(bar(kBarKVEmpty + s), ((pos / C::kQStages) & 1) ^ 1, ctl)) {
            ok = false;
            break;
          }
          // K(t) and V(t) land on the full barrier of K(t)'s stage (an even stage)
          const int sf = (2 * t) % C::kQStages;
          if (kind == 0) mbar_arrive_expect_tx(bar(kBarKVFull + sf), 2 * C::kTileBytes);
#pragma unroll
          for (int hf = 0; hf < C::kHalves; ++hf)
            tma_load_4d(sb + C::kQKVOff + s * C::kTileBytes + hf * C::kAtomBytes,
                        kind ? &tm_v : &tm_k, bar(kBarKVFull + sf), 64 * hf, g, 128 * (jlo + t), b);
          issued = pos + 1;
        }
      }
      volatile int zero = 0;
      const WaitCtl drain_ctl{&zero, p.timeout_ns};
      mbar_wait(bar(kBarIn), 0, drain_ctl);
      for (int s = 0; s < C::kQStages && s < issued; s += 2) {
        const int lastp = s + C::kQStages * ((issued - 1 - s) / C::kQStages);
        mbar_wait(bar(kBarKVFull + s), (lastp / C::kQStages) & 1, drain_ctl);
      }
    }
  } else if (warp == 9) {
    // ============ MMA issuer ============
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, false);
      constexpr uint32_t idesc_acc = idesc_bf16_f32(128, D, true);
      auto mma_rows = [&](uint32_t d, uint32_t a, uint32_t bt) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t o2 = (kk / 4) * C::kAtomBytes + (kk % 4) * 32;
          umma_ss(tmem + d, smem_desc_sw128(a + o2, 16, 1024), smem_desc_sw128(bt + o2, 16, 1024),
                  idesc_s, kk > 0 ? 1u : 0u);
        }
      };
      // K(t) and V(t) in shared memory (one barrier for both).  The MMAs read them through
      // the async proxy that wrote them; no tcgen05 fence is needed after this wait.
      auto kv_wait = [&](int pos) {
        return mbar_wait(bar(kBarKVFull + pos % C::kQStages), (pos / C::kQStages) & 1, ctl);
      };
      // Order: S(0) dP(0) | S(t+1) dP(t+1) once S(t), dP(t) are in registers | dQ(t) once
      // dS(t) is in TMEM: the next tile's products overlap the elementwise work on this one.
      auto tile_addr = [&](int pos) {
        return sb + C::kQKVOff + (pos % C::kQStages) * C::kTileBytes;
      };
      auto issue_sdp = [&](int t) -> bool {
        if (!kv_wait(2 * t)) return false;
        mma_rows(colS, sb + C::kQOff, tile_addr(2 * t));       // S = Q K^T
        mma_rows(colDP, sb + C::kDOOff, tile_addr(2 * t + 1));  // dP = dO V^T
        tc_commit(bar(kBarSDP));
        tc_commit(bar(kBarKVEmpty + (2 * t + 1) % C::kQStages));  // V(t) is done
        return true;
      };
      bool ok = n_kt > 0 && mbar_wait(bar(kBarIn), 0, ctl);
      tc_fence_after();
      if (ok) ok = issue_sdp(0);
      for (int t = 0; t < n_kt && ok; ++t) {
        if (t + 1 < n_kt) {
          if (!(ok = mbar_wait(bar(kBarFree), t & 1, ctl))) break;
          tc_fence_after();
          if (!(ok = issue_sdp(t + 1))) break;
        }
        if (!(ok = mbar_wait(bar(kBarDS), t & 1, ctl))) break;
        tc_fence_after();
        // dQ += dS K (K tile as the MN-major B operand)
        const uint32_t kt = tile_addr(2 * t);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_ts(tmem + colDQ, tmem + colDS + kk * 8,
                  smem_desc_sw128(kt + kk * 16 * 128, C::kAtomBytes, 1024), idesc_acc,
                  (t == 0 && kk == 0) ? 0u : 1u);
        tc_commit(bar(kBarDQ));
        tc_commit(bar(kBarKVEmpty + (2 * t) % C::kQStages));
      }
      tc_commit(bar(kBarO));
      tc_commit(bar(kBarDrain));
      volatile int zero = 0;
      const WaitCtl drain_ctl{&zero, p.timeout_ns};
      mbar_wait(bar(kBarDrain), 0, drain_ctl);
    }
  } else {
    // ============ elementwise: thread = Q row; this warp's half of the key columns ============
    const int wq = warp & 3, ch = warp >> 2;
    const int r = 32 * wq + lane;
    const int i = tok0 + r / p.Gp;
    const int hh = h0 + r % p.Gp;
    const uint32_t trow = tmem + (static_cast<uint32_t>(32 * wq) << 16);
    const uint64_t sl2 = f2(p.scale_log2, p.scale_log2);
    const size_t vrow = (static_cast<size_t>(b) * p.Hq + hh) * p.Sq_pad + min(i, p.Sq_pad - 1);
    const float nl2 = p.lse2[vrow], ndl = p.delta[vrow];  // -L log2(e), -D
    const uint64_t nl2x2 = f2(nl2, nl2), ndlx2 = f2(ndl, ndl);
    const int ip = i + off;
    const int my_lo = p.window > 0 ? max(0, ip - p.window + 1) : 0;
    const int my_hi = p.causal ? min(ip, p.Skv - 1) : p.Skv - 1;
    // rows of the tile that bound its masks (all rows of a tile share the key-tile range)
    const int lo_last = p.window > 0 ? max(0, last + off - p.window + 1) : 0;
    const int hi_first = p.causal ? min(first + off, p.Skv - 1) : p.Skv - 1;
    for (int t = 0; t < n_kt; ++t) {
      const int j = jlo + t;
      bool ok = mbar_wait(bar(kBarSDP), t & 1, ctl);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      const bool need_mask = (128 * j < lo_last) || (128 * j + 127 > hi_first) || i >= p.Sq;
      uint32_t ds[32];
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        uint32_t sv[32], dv[32];
        tmem_ld32(trow + colS + 64 * ch + 32 * cc, sv);
        tmem_ld32(trow + colDP + 64 * ch + 32 * cc, dv);
        tmem_wait_ld();
#pragma unroll
        for (int x = 0; x < 16; ++x) {
          float a0, a1;
          f2_split(f2_fma(f2(__uint_as_float(sv[2 * x]), __uint_as_float(sv[2 * x + 1])), sl2,
                          nl2x2), a0, a1);
          float p0 = ex2(a0), p1 = ex2(a1);
          if (need_mask) {
            const int key = 128 * j + 64 * ch + 32 * cc + 2 * x;
            if (key < my_lo || key > my_hi || i >= p.Sq) p0 = 0.f;
            if (key + 1 < my_lo || key + 1 > my_hi || i >= p.Sq) p1 = 0.f;
          }
          float d0, d1;
          f2_split(f2_mul(f2(p0, p1), f2_add(f2(__uint_as_float(dv[2 * x]),
                                                 __uint_as_float(dv[2 * x + 1])), ndlx2)),
                   d0, d1);
          ds[16 * cc + x] = pack_bf16x2(d0, d1);
        }
      }
      // S and dP of this tile have been read: the next tile's products may start
      tc_fence_before();
      mbar_arrive(bar(kBarFree));
      // the previous dQ product has read its dS before this one is written over it
      if (t > 0) {
        ok = mbar_wait(bar(kBarDQ), (t - 1) & 1, ctl);
        if (!__all_sync(0xffffffffu, ok)) break;
        tc_fence_after();
      }
      tmem_st32(trow + colDS + 32 * ch, ds);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(kBarDS));
    }
    // ---- epilogue: scale * dQ -> bf16 -> swizzled smem (the Q tile) -> TMA; warps 0-3 take
    // the first half of the head dims, warps 4-7 the second ----
    bool have = false;
    if (n_kt > 0) {
      bool ok = mbar_wait(bar(kBarO), 0, ctl);
      have = __all_sync(0xffffffffu, ok);
      tc_fence_after();
    }
    uint8_t* stage = smem + C::kQOff;
#pragma unroll
    for (int cc = 0; cc < D / 64; ++cc) {
      const int c = ch * (D / 64) + cc;
      uint32_t ov[32];
      if (have) {
        tmem_ld32(trow + colDQ + 32 * c, ov);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int x = 0; x < 32; ++x) ov[x] = 0u;
      }
      const int hf = c >> 1;
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        uint4 w;
        w.x = pack_bf16x2(__uint_as_float(ov[8 * q4 + 0]) * p.scale, __uint_as_float(ov[8 * q4 + 1]) * p.scale);
        w.y = pack_bf16x2(__uint_as_float(ov[8 * q4 + 2]) * p.scale, __uint_as_float(ov[8 * q4 + 3]) * p.scale);
        w.z = pack_bf16x2(__uint_as_float(ov[8 * q4 + 4]) * p.scale, __uint_as_float(ov[8 * q4 + 5]) * p.scale);
        w.w = pack_bf16x2(__uint_as_float(ov[8 * q4 + 6]) * p.scale, __uint_as_float(ov[8 * q4 + 7]) * p.scale);
        const int chunk = ((c & 1) * 4 + q4) ^ (r & 7);
        *reinterpret_cast<uint4*>(stage + hf * C::kAtomBytes + r * 128 + chunk * 16) = w;
      }
    }
    fence_proxy_async_smem();
    named_bar_sync(1, 256);
    if (threadIdx.x == 0 && tok0 < p.Sq) {
#pragma unroll
      for (int hf = 0; hf < C::kHalves; ++hf)
        tma_store_4d(&tm_dq, sb + C::kQOff + hf * C::kAtomBytes, 64 * hf, h0, tok0, b);
      tma_store_commit();
      tma_store_wait_read_all();
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
