// Attention backward pass for sm_100a.
//
// The forward pass keeps only O and the row log-sum-exp; the backward pass recomputes the
// probabilities tile by tile instead of storing them ("FlashAttention on Ascend NPUs",
// recomputation section).  With L the row log-sum-exp and D_i = dO_i . O_i:
//   P_ij = exp(scale q_i.k_j - L_i),  dP_ij = dO_i . v_j,  dS_ij = P_ij (dP_ij - D_i)
//   dV_j = sum_i P_ij dO_i,  dK_j = scale sum_i dS_ij q_i,  dQ_i = scale sum_j dS_ij k_j
// Three kernels:
//   fa_bwd_prep_kernel   -D_i and -L_i * log2(e) per (b, h, i) into a padded workspace
//                        (padding rows get L = +inf, D = 0: they contribute nothing), and the
//                        row's fp32 dQ accumulator set to zero;
//   fa_bwd_kernel        one CTA per (b, KV head, 128-key tile): per (query head of the group,
//                        128-query tile) S^T = K Q^T and dP^T = V dO^T, then dV += P^T dO,
//                        dK += dS^T Q (GQA heads summed in TMEM, one bf16 store of dK and dV at
//                        the end) and the tile's share of dQ, dS K, staged in the unit's own
//                        (no longer read) Q and dO buffers and added into the fp32 accumulator
//                        by TMA tensor reductions (so S and dP are computed once per (query,
//                        key) tile);
//   fa_bwd_dq_finalize_kernel  dQ = scale * accumulator, rounded to bf16.
// dK and dV are deterministic; dQ sums the key tiles' shares in the order the reductions land.
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
  int n_tiles;         // key tiles
  float scale;         // softmax scale
  float scale_log2;    // scale * log2(e)
  int causal, window;
  const uint16_t* o;     // bf16 [B, Sq, Hq, D]
  const uint16_t* dout;  // bf16 [B, Sq, Hq, D]
  const float* lse;      // natural log [B, Hq, Sq]
  float* lse2;           // workspace [B * Hq, Sq_pad]: -L * log2(e)
  float* delta;          // workspace [B * Hq, Sq_pad]: -D
  float* dq_acc;         // workspace [B, Sq, Hq, D] fp32: sum over key tiles of dS K
  uint16_t* dq;          // bf16 [B, Sq, Hq, D] output
  uint64_t timeout_ns;
};

template <int D>
struct BwdCfg {
  static constexpr int kThreads = 320;
  static constexpr int kHalves = D / 64;
  static constexpr int kAtomBytes = 128 * 128;
  static constexpr int kTileBytes = 128 * D * 2;
  static constexpr uint32_t kTmemCols = 512;
  // K and V tiles, then a ring of (Q, dO, L, D) units
  static constexpr int kUStages = (D == 128) ? 2 : 4;
  static constexpr int kUnitBytes = 2 * kTileBytes + 2 * 128 * 4;
  static constexpr int kKOff = 0;
  static constexpr int kVOff = kTileBytes;
  static constexpr int kUOff = 2 * kTileBytes;
  // dS^T (bf16, 128 keys x 128 queries as two 128-byte swizzle atoms of 64 queries) is the A
  // operand of dK += dS^T Q (K-major) and of dQ = dS K (read MN-major); it has a buffer of its
  // own.  A unit's dQ share (128 query rows x D fp32) is then staged for the TMA reductions in
  // two halves: dims [0, D/2) over the unit's dO tile, dims [D/2, D) over the dS^T buffer (both
  // free once dK, the last product reading them, has run).
  static constexpr int kDSOff = kUOff + kUStages * kUnitBytes;
  static constexpr int kStgBytes = 128 * (D / 2) * 4;
  static_assert(kStgBytes <= 2 * kAtomBytes, "dQ staging half over the dS^T buffer");
  static constexpr int kUBarOff = kDSOff + 2 * kAtomBytes;
  // barriers: kv_full, u_full[S] (Q and the vectors), q_empty[S], s_full, dp_full, p_ready,
  // ds_ready, o_final, drain, u_do[S] (dO), dq_full, dq_free, dk_done, do_empty[S], x_free
  static constexpr int kUNumBars = 11 + 4 * kUStages;
  static constexpr int kUMiscOff = kUBarOff + 8 * kUNumBars;
  // (no slack for aligning the base: the kernel requires the dynamic shared memory to start
  // 1024-byte aligned, checks it and reports a device error otherwise)
  static constexpr int kUSmemBytes = kUMiscOff + 16;
  static_assert(kUSmemBytes <= 227 * 1024, "backward kernel over the shared memory");
};

// ---------------------------------------------------------------------------------------
// -D_i = -dO_i . O_i and -L_i * log2(e) per (b, h, i) row, D / 8 lanes per row (stored negated
// so the kernels add them); padding rows past Sq get L = +inf and D = 0.  Rows with L = -inf (no
// visible key) also get +inf: their P is 0.  The row's dQ accumulator is zeroed.
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
  // this row's fp32 dQ accumulator starts at zero (8 floats per lane)
  if (valid && i < p.Sq) {
    float4* z = reinterpret_cast<float4*>(
        p.dq_acc + ((static_cast<size_t>(b) * p.Sq + i) * p.Hq + h) * D + 8 * sub);
    z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
    z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
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
// One CTA per (b, KV head g, key tile j): dK and dV of the tile, and its share of dQ.
// ---------------------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(320, 1)
    fa_bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v,
                  const __grid_constant__ CUtensorMap tm_do,
                  const __grid_constant__ CUtensorMap tm_vec,
                  const __grid_constant__ CUtensorMap tm_dk,
                  const __grid_constant__ CUtensorMap tm_dv,
                  const __grid_constant__ CUtensorMap tm_dqacc, const BwdParams p) {
  using C = BwdCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 128-byte swizzled TMA boxes need 1024-byte aligned shared memory, and this kernel has no
  // room to align the base itself
  if ((smem_u32(smem_raw) & 1023u) != 0) {
    if (threadIdx.x == 0) atomicOr(&g_fa_device_status, kDevStatusLayout);
    return;
  }
  uint8_t* smem = smem_raw;
  const uint32_t sb = smem_u32(smem);
  auto bar = [&](int idx) { return sb + C::kUBarOff + 8u * idx; };
  constexpr int kBarKV = 0, kBarUFull = 1, kBarUEmpty = 1 + C::kUStages;
  constexpr int kBarS = 1 + 2 * C::kUStages, kBarDP = kBarS + 1, kBarP = kBarS + 2,
                kBarDS = kBarS + 3, kBarO = kBarS + 4, kBarDrain = kBarS + 5,
                kBarUDo = kBarS + 6, kBarDQFull = kBarUDo + C::kUStages,
                kBarDQFree = kBarDQFull + 1, kBarDKDone = kBarDQFull + 2,
                kBarDOEmpty = kBarDQFull + 3, kBarXFree = kBarDOEmpty + C::kUStages;
  static_assert(kBarXFree + 1 == C::kUNumBars, "barrier count");
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
      mbar_init(bar(x), (x == kBarP || x == kBarDS || x == kBarDQFree) ? 256
                        : ((x >= kBarDOEmpty && x < kBarDOEmpty + C::kUStages) || x == kBarXFree)
                            ? 8
                            : 1);
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
  // dQ of a unit accumulates over dP^T's columns once the elementwise warps have read dP^T
  constexpr uint32_t colS = 0, colDP = 128, colDQ = 128, colDV = 256, colDK = 256 + D;

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
        // Q and the vectors are free once dK of the stage's previous unit has run; dO (which
        // also held that unit's dS^T and half its dQ staging) once the reductions have read it
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
        // (copies in flight from here on are waited for below, even if dO is never started:
        // that wait then runs out)
        issued = u + 1;
        if (u >= C::kUStages &&
            !mbar_wait(bar(kBarDOEmpty + s), ((u / C::kUStages) - 1) & 1, ctl))
          break;
        mbar_arrive_expect_tx(bar(kBarUDo + s), C::kTileBytes);
#pragma unroll
        for (int hf = 0; hf < C::kHalves; ++hf)
          tma_load_4d(base + C::kTileBytes + hf * C::kAtomBytes, &tm_do, bar(kBarUDo + s),
                      64 * hf, h, i0, b);
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
      // A K-major (or in TMEM), B MN-major
      constexpr uint32_t idesc_acc = idesc_bf16_f32(128, D, true);
      // A and B both MN-major (bit 15: A major)
      constexpr uint32_t idesc_dq = idesc_bf16_f32(128, D, true) | (1u << 15);
      // D[tmem] = A_tile (K-major rows) . B_tile^T, K = D
      auto mma_rows = [&](uint32_t d, uint32_t a, uint32_t bt) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t o2 = (kk / 4) * C::kAtomBytes + (kk % 4) * 32;
          umma_ss(tmem + d, smem_desc_sw128(a + o2, 16, 1024), smem_desc_sw128(bt + o2, 16, 1024),
                  idesc_s, kk > 0 ? 1u : 0u);
        }
      };
      // dV += P^T dO: A = P^T in TMEM (queries 0-63 in columns [colS, colS + 32), queries
      // 64-127 in [colS + 64, colS + 96)), B = the dO tile (MN-major, K = its 128 rows)
      auto mma_dv = [&](uint32_t dot, bool first) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_ts(tmem + colDV, tmem + colS + 64 * (kk / 4) + 8 * (kk % 4),
                  smem_desc_sw128(dot + kk * 16 * 128, C::kAtomBytes, 1024), idesc_acc,
                  (first && kk == 0) ? 0u : 1u);
      };
      // dK += dS^T Q: A = dS^T (K-major: key rows, 16 queries per step), B = the Q tile
      // (MN-major, K = its 128 rows)
      auto mma_dk = [&](uint32_t ds, uint32_t qt, bool first) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_ss(tmem + colDK,
                  smem_desc_sw128(ds + (kk / 4) * C::kAtomBytes + (kk % 4) * 32, 16, 1024),
                  smem_desc_sw128(qt + kk * 16 * 128, C::kAtomBytes, 1024), idesc_acc,
                  (first && kk == 0) ? 0u : 1u);
      };
      // dQ = dS K over this key tile: A = dS (MN-major: the dS^T tile read with the queries
      // contiguous, 16 keys per step), B = the K tile (MN-major, K = its 128 key rows)
      auto mma_dq = [&](uint32_t ds) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_ss(tmem + colDQ, smem_desc_sw128(ds + kk * 16 * 128, C::kAtomBytes, 1024),
                  smem_desc_sw128(sb + C::kKOff + kk * 16 * 128, C::kAtomBytes, 1024), idesc_dq,
                  kk > 0 ? 1u : 0u);
      };
      // Order: S(0) dP(0) | dV(u) S(u+1) dQ(u) dK(u) dP(u+1) | ...: the tensor core works on the
      // next unit's S while the elementwise warps turn dP into dS; dQ(u) goes first so that its
      // read-out overlaps dK(u); dP(u+1) waits until dQ(u) (which shares its columns) has been
      // read out.
      auto unit_tiles = [&](int u, uint32_t& qt, uint32_t& dot) {
        qt = sb + C::kUOff + (u % C::kUStages) * C::kUnitBytes;
        dot = qt + C::kTileBytes;
      };
      // (waits on copies into shared memory need no tcgen05 fence: the MMAs read through the
      // async proxy that wrote them; waits on TMEM or shared memory written by other warps do)
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
        mma_dv(dot, u == 0);                  // dV += P^T dO
        if (nxt) {
          if (!(ok = mbar_wait(bar(kBarUFull + (u + 1) % C::kUStages), ((u + 1) / C::kUStages) & 1, ctl)))
            break;
          unit_tiles(u + 1, qn, don);
          mma_rows(colS, sb + C::kKOff, qn);  // S^T of the next unit (after dV read P)
          tc_commit(bar(kBarS));
        }
        if (!(ok = mbar_wait(bar(kBarDS), u & 1, ctl))) break;
        tc_fence_after();
        const uint32_t ds = sb + C::kDSOff;
        mma_dq(ds);                           // this tile's dQ share = dS K
        tc_commit(bar(kBarDQFull));
        mma_dk(ds, qt, u == 0);               // dK += dS^T Q
        tc_commit(bar(kBarDKDone));
        tc_commit(bar(kBarUEmpty + u % C::kUStages));  // Q (the elementwise warps free dO)
        if (nxt) {
          if (!(ok = mbar_wait(bar(kBarDQFree), u & 1, ctl))) break;
          tc_fence_after();
          if (!(ok = mbar_wait(bar(kBarUDo + (u + 1) % C::kUStages), ((u + 1) / C::kUStages) & 1, ctl)))
            break;
          mma_rows(colDP, sb + C::kVOff, don);  // dP^T of the next unit (after dQ was read)
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
    // ============ elementwise: thread = key row (S^T, dP^T) / query row (dQ); this warp's
    // half of the columns ============
    const int wq = warp & 3, ch = warp >> 2;
    const int r = 32 * wq + lane;
    const int key = k0 + r;
    const uint32_t trow = tmem + (static_cast<uint32_t>(32 * wq) << 16);
    const uint64_t sl2 = f2(p.scale_log2, p.scale_log2);
    // Lane 0: the stage whose dQ reductions were issued last and whose release to the producer
    // waits until the reductions have read it (done after the next unit's P, so the reductions
    // overlap that work), or -1.
    int pend_s = -1;
    auto release_pending = [&]() {
      if (lane == 0 && pend_s >= 0) {
        tma_store_wait_read_all();
        mbar_arrive(bar(kBarDOEmpty + pend_s));
      }
      pend_s = -1;
    };
    for (int u = 0; u < n_units; ++u) {
      const int s = u % C::kUStages;
      const int h = g * p.G + u / n_qt;
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
      release_pending();
      if (lane == 0) mbar_arrive(bar(kBarXFree));  // this warp's earlier reductions were read
      // ---- dS = P (dP^T - D), bf16, into shared memory as row r (key) of the dS^T tile ----
      ok = mbar_wait(bar(kBarDP), u & 1, ctl);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      uint32_t ds[32];
      {
        uint32_t dv[64];
        tmem_ld32(trow + colDP + 64 * ch, *reinterpret_cast<uint32_t(*)[32]>(dv));
        tmem_ld32(trow + colDP + 64 * ch + 32, *reinterpret_cast<uint32_t(*)[32]>(dv + 32));
        tmem_wait_ld();
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
      }
      // the dS^T buffer held the previous unit's dQ staging: every warp's reductions of it
      // have been read (each warp's lane 0 waited in release_pending) before anyone writes
      ok = mbar_wait(bar(kBarXFree), u & 1, ctl);
      if (!__all_sync(0xffffffffu, ok)) break;
      {
        // atom ch holds queries 64 ch .. 64 ch + 63; 16-byte chunk c of row r (queries
        // 8c .. 8c + 7 of the atom) sits at chunk c ^ (r & 7), the 128-byte swizzle
        uint8_t* row_ptr = smem + C::kDSOff + ch * C::kAtomBytes + r * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c)
          *reinterpret_cast<uint4*>(row_ptr + 16 * (c ^ (r & 7))) =
              make_uint4(ds[4 * c], ds[4 * c + 1], ds[4 * c + 2], ds[4 * c + 3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(bar(kBarDS));
      // ---- this unit's dQ share: TMEM lane = query row r, this warp's half of the dims ----
      ok = mbar_wait(bar(kBarDQFull), u & 1, ctl);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      uint32_t qv[D / 2];
#pragma unroll
      for (int c = 0; c < D / 64; ++c)
        tmem_ld32(trow + colDQ + (D / 2) * ch + 32 * c,
                  *reinterpret_cast<uint32_t(*)[32]>(qv + 32 * c));
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(bar(kBarDQFree));
      // the staging of ch = 1 goes over dS^T, which dK += dS^T Q reads (ch = 0 stages over dO,
      // which dP and dV finished reading before dS was computed)
      if (ch) {
        ok = mbar_wait(bar(kBarDKDone), u & 1, ctl);
        if (!__all_sync(0xffffffffu, ok)) break;
      }
      {
        // Stage this warp's 32 rows x D/2 dims: boxes of 32 rows x 32 fp32 (128 bytes a row,
        // 128-byte swizzle), box (wq, k) at 4 KB * (k * 4 + wq) of the unit's dO tile (ch = 0)
        // or of the dS^T buffer (ch = 1), which every product has finished reading (dK is the
        // last); then one lane adds them into the accumulator (the dO tile goes back to the
        // producer once they are read).
        constexpr int kBoxes = D / 64;
        const uint32_t st_base =
            ch ? C::kDSOff : C::kUOff + s * C::kUnitBytes + C::kTileBytes;
#pragma unroll
        for (int k = 0; k < kBoxes; ++k) {
          uint8_t* row_ptr = smem + st_base + 4096 * (k * 4 + wq) + lane * 128;
#pragma unroll
          for (int c = 0; c < 8; ++c)
            *reinterpret_cast<uint4*>(row_ptr + 16 * (c ^ (lane & 7))) =
                make_uint4(qv[32 * k + 4 * c], qv[32 * k + 4 * c + 1], qv[32 * k + 4 * c + 2],
                           qv[32 * k + 4 * c + 3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          const int t0 = i0 + 32 * wq;  // first query row of this warp
          if (t0 < p.Sq) {
#pragma unroll
            for (int k = 0; k < kBoxes; ++k)
              tma_reduce_add_4d(&tm_dqacc, sb + st_base + 4096 * (k * 4 + wq),
                                (D / 2) * ch + 32 * k, h, t0, b);
            tma_store_commit();
          }
        }
        pend_s = s;
        __syncwarp();
      }
    }
    release_pending();
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
// dQ = scale * accumulator -> bf16, eight elements per thread.
// ---------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) fa_bwd_dq_finalize_kernel(const float* acc, uint16_t* dq,
                                                                 float scale, long long n8) {
  const long long t = static_cast<long long>(blockIdx.x) * 256 + threadIdx.x;
  if (t >= n8) return;
  const float4* a = reinterpret_cast<const float4*>(acc) + 2 * t;
  const float4 x = a[0], y = a[1];
  uint4 w;
  w.x = pack_bf16x2(x.x * scale, x.y * scale);
  w.y = pack_bf16x2(x.z * scale, x.w * scale);
  w.z = pack_bf16x2(y.x * scale, y.y * scale);
  w.w = pack_bf16x2(y.z * scale, y.w * scale);
  reinterpret_cast<uint4*>(dq)[t] = w;
}

}  // namespace fa
