// bwd.cu -- the two backward kernels of sigmoid attention for sm_100a.
//
// The backward pass is split in two kernels, one for dQ and one for dK/dV, so
// that every output block has exactly one owner and no atomics are needed; the
// attention weights are recomputed in-kernel instead of being stored (Better
// Models, Faster Training: Sigmoid Attention for single-cell Foundation
// Models, sec. 2C "backward decomposition"). The sigmoid's derivative is
// sigma' = sigma (1 - sigma) (sec. 2B) and its Jacobian is diagonal, so
//
//   dP = dO V^T,  dS = dP * P * (1 - P)   (elementwise; no row-sum pre-pass),
//   dQ = scale * dS K,  dK = scale * dS^T Q,  dV = P^T dO.
//
// Both kernels are one template. A work item is a block of 128 "rows" of one
// (b, h); the kernel streams 128-wide blocks of "columns" of the same slice:
//
//              rows  R1  R2  | columns C1  C2 | S        dP        accumulators
//   dQ   (KV=0) queries Q  dO |        K   V  | Q K^T    dO V^T    A1 += dS K      -> dQ
//   dK/dV(KV=1) keys    K  V  |        Q   dO | K Q^T    V dO^T    A1 += dS^T Q    -> dK
//                                                                   A2 += P^T dO    -> dV
//
// Per block j of BN columns, in tensor memory (TMEM):
//   XS  = R1 C1_j^T  (S,  fp32)  -> epilogue: P = sigma(S*scale + b), 0 for
//                                   padded columns; bf16 P to its own region
//   XdP = R2 C2_j^T  (dP, fp32)  -> epilogue: dS = dP P (1 - P); bf16 dS to
//                                   its own region
//   A1 += dS C1_j, A2 += P C2_j  (A operand read from TMEM, per 32-column chunk)
// (The kernels hold -P and -dS in TMEM and accumulate -dQ / scale, -dK / scale
// and -dV, and the readout multiplies by -scale and -1: the negated forms come
// out of the sigmoid's polynomial without a sign flip per score.)
// A region is released as soon as the epilogue has copied it to registers, so
// the products of block j+1 overlap the epilogue of block j. One thread issues
// a tcgen05.mma only every ~100 cycles, so the products are spread over four
// issuing warps (S, dP, A1, A2), each with its own TMEM region. C1 and C2 have
// rings of their own.
//
// BN is 128, except for dK/dV at D = 128, where the two D-wide accumulators
// leave room in the 512 TMEM columns only for 64-column S and dP regions:
//   XS [0,BN) XdP [BN,2BN) P [2BN,2.5BN) dS [2.5BN,3BN) A1 [3BN,3BN+D) A2 after.
// Warps: 0 .. E-1 epilogue, E = 4 G with G column groups (warps 4g..4g+3 take
// columns [g BN/G, (g+1) BN/G) of each block, in chunks of CW = 32 columns;
// G = 4, or 2 for dK/dV at D = 128), then the TMA
// producer (also claims the work items and passes them on through the
// shared-memory item ring; for dQ at D = 64 over padded inputs it also writes
// the zeros of the rows no item covers, with bulk copies from shared memory
// while the compute runs), the S issuer (owns TMEM), the dP issuer, the A1
// issuer and (dK/dV) the A2 issuer; idle warps round the CTA up to whole
// warpgroups. PACKED selects the input layout, as in the forward kernel.
#include "common.cuh"

namespace sigattn {

template <int D, bool KV>
struct BwdCfg {
  static constexpr int BM = kBwdItemRows;   // 128 rows per item
  static constexpr int BN = bwd_col_block(KV, D);
  // Epilogue column groups (warps per lane quadrant) and chunk width: 16
  // epilogue warps on 32-column chunks, except dK/dV at D = 128 (8 warps:
  // its 64-column blocks would leave 16 warps 16-column chunks, measured
  // slower: 0.918 -> 0.984 ms on the dense d = 128 workload).
  static constexpr int GROUPS = (D == 64 || !KV) ? 4 : 2;
  // dQ at D = 64: a warp whose columns of a block hold no valid score (keys
  // past the sequence's end, or padded rows only) skips the block's reads and
  // sigmoids and writes zeros (75 %-padded sweep 0.1756 -> 0.1716 ms,
  // scRNA-shaped 0.0973 -> 0.0952 ms, long_8k 0.0584 -> 0.0563 ms). The same
  // path in the dK/dV kernel and at D = 128 made those kernels slower, even
  // where no such block occurs.
  static constexpr bool SKIP_DEAD = (!KV && D == 64);
  // sigma and sigma' are carried negated (the tail polynomial run with
  // negated coefficients gives -sigma, and -sigma' = (-sigma)^2 + (-sigma) is
  // one packed FMA), so the kernel writes -P and -dS, its accumulators hold
  // -dQ / scale, or -dK / scale and -dV, and the readout multiplies by -scale
  // and -1: no sign flip per score. Interleaved runs: 0 %-padded dQ 1.664 ->
  // 1.598 ms and dK/dV 1.958 -> 1.853 ms, dense_d128 dQ 0.649 -> 0.640 ms and
  // dK/dV 0.949 -> 0.936 ms.
  static constexpr bool NEG_SLOPE = true;
  // Blocks before the last run without masking code (a second instance of
  // the block's code): dQ 0 %-padded 1.599 -> 1.552 ms, 75 % 0.1647 ->
  // 0.1602 ms, dense_d128 0.663 -> 0.657 ms; dK/dV at D = 128 0.934 ->
  // 0.929 ms. The dK/dV kernel at D = 64 spills with two instances (1.854 ->
  // 1.912 ms) and runs every block in the masking form.
  static constexpr bool SPLIT_MASK = !(KV && D == 64);
  static constexpr int CW = 32;
  static constexpr int NCH = BN / CW;       // chunks per block
  static constexpr int CPW = NCH / GROUPS;  // chunks per epilogue warp
  static_assert(CPW >= 1 && NCH <= 4, "chunking");
  static constexpr int BOX_R = 128 * 64 * 2;   // [128 rows][64 cols] bf16
  static constexpr int BOX_C = BN * 64 * 2;    // [BN rows][64 cols] bf16
  static constexpr int TILE_R = 128 * D * 2;
  static constexpr int TILE_C = BN * D * 2;
  static constexpr int ST1 = (D == 128 && BN == 128) ? 3 : 4;   // C1 ring slots
  static constexpr int ST2 = (D == 128 && BN == 128) ? 2 : 4;   // C2 ring slots
  static constexpr int OFF_R1 = 0;
  static constexpr int OFF_R2 = TILE_R;
  static constexpr int OFF_C1 = 2 * TILE_R;
  static constexpr int OFF_C2 = OFF_C1 + ST1 * TILE_C;
  // dQ at D = 64 over padded inputs: a 16 KB block of zeros in shared memory
  // from which the producer writes the padded rows of dQ with bulk copies
  // while the compute runs (at D = 128 the rings leave no room for it).
  static constexpr int ZBUF = (!KV && D == 64) ? 16384 : 0;
  static constexpr int OFF_Z = OFF_C2 + ST2 * TILE_C;
  static constexpr int SMEM_BYTES = OFF_Z + ZBUF;
  static constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;
  static constexpr int TM_XS = 0;
  static constexpr int TM_XDP = BN;
  static constexpr int TM_P = 2 * BN;
  static constexpr int TM_DS = 2 * BN + BN / 2;
  static constexpr int TM_A1 = 3 * BN;
  static constexpr int TM_A2 = 3 * BN + D;
  static constexpr int TMEM_COLS = 512;
  static_assert(TM_A1 + (KV ? 2 : 1) * D <= TMEM_COLS, "TMEM budget");
  // A second dP region where the columns allow (dK/dV at D = 128): the dP
  // products of block j+1 need not wait for the epilogue to copy out dP(j).
  static constexpr int TM_XDP1 = TM_A1 + (KV ? 2 : 1) * D;
  static constexpr int NXDP = (TM_XDP1 + BN <= TMEM_COLS) ? 2 : 1;
  static_assert(SMEM_ALLOC <= 227 * 1024 - 1024, "shared memory budget");
  static constexpr int EPI_WARPS = 4 * GROUPS;
  static constexpr int ISSUERS = KV ? 4 : 3;
  // Whole warpgroups: the epilogue's, then one or two holding the producer,
  // the issuers and idle warps. The single-thread roles give registers to the
  // epilogue (setmaxnreg). The launch gives every thread LAUNCH_REGS; the
  // split must not exceed that total (the launcher also checks it against
  // the count the compiler actually allocated).
  static constexpr int WARPS = (EPI_WARPS + 1 + ISSUERS + 3) / 4 * 4 < 16 ? 16 : (EPI_WARPS + 1 + ISSUERS + 3) / 4 * 4;
  static constexpr int THREADS = WARPS * 32;
  static constexpr int LAUNCH_REGS = (65536 / THREADS) / 8 * 8;
  static constexpr int OTHER_REGS = WARPS > 20 ? 48 : WARPS > 16 ? 56 : 64;
  static constexpr int EPI_REGS =
      ((LAUNCH_REGS * WARPS - OTHER_REGS * (WARPS - EPI_WARPS)) / EPI_WARPS) / 8 * 8 > 184
          ? 184
          : ((LAUNCH_REGS * WARPS - OTHER_REGS * (WARPS - EPI_WARPS)) / EPI_WARPS) / 8 * 8;
  static_assert(EPI_REGS * EPI_WARPS + OTHER_REGS * (WARPS - EPI_WARPS) <= LAUNCH_REGS * WARPS, "register split");
  static_assert(EPI_REGS >= LAUNCH_REGS && OTHER_REGS <= LAUNCH_REGS, "setmaxnreg directions");
};

template <int ST1, int ST2>
struct BwdBarriers {
  uint64_t r_full, r_empty;
  uint64_t c1_full[ST1], c1_empty[ST1];
  uint64_t c2_full[ST2], c2_empty[ST2];
  uint64_t xs_full, xdp_full[2];   // S / dP of the current block are in TMEM
  uint64_t xs_read, xdp_read[2];   // the epilogue has copied S / dP out (per dP region)
  uint64_t p_full[4], ds_full[4];  // bf16 P / dS of a 32-column chunk written
  uint64_t p_free, ds_free;        // the accumulation products of a block have read P / dS
  uint64_t acc_full, acc_empty;
  uint64_t drain[4];
  ItemRing ring;
  uint32_t tmem_base;
  int abort;
};

// kr: the keys the call covers (whole sequences: {0, Lmax}). For dQ the
// columns are the range's keys; for dK/dV the rows are, and L is then the
// rows per (b, h) slice of the dK/dV outputs (kr.count). F32OUT (dQ only):
// write dQ as the fp32 partial sum over the range's keys.
template <int D, bool KV, bool PACKED, bool F32OUT>
__global__ void __launch_bounds__(BwdCfg<D, KV>::THREADS, 1)
    bwd_kernel(const __grid_constant__ CUtensorMap tm_r1, const __grid_constant__ CUtensorMap tm_r2,
               const __grid_constant__ CUtensorMap tm_c1, const __grid_constant__ CUtensorMap tm_c2,
               void* __restrict__ out1, void* __restrict__ out2, int* __restrict__ ws, int H, int L, KeyRange kr,
               const int* __restrict__ fill_lengths, int B, int len_bound, int fill_parts, int* __restrict__ err,
               int overlap) {
  using C = BwdCfg<D, KV>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ BwdBarriers<C::ST1, C::ST2> bar;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  volatile int* abort_flag = &bar.abort;
  constexpr int kProducerWarp = C::EPI_WARPS;
  constexpr int kSWarp = C::EPI_WARPS + 1;
  constexpr int kDPWarp = C::EPI_WARPS + 2;
  constexpr int kA1Warp = C::EPI_WARPS + 3;
  constexpr int kA2Warp = KV ? C::EPI_WARPS + 4 : -1;

  if (threadIdx.x == 0) {
    mbar_init(&bar.r_full, 1);
    mbar_init(&bar.r_empty, 2);  // S issuer (R1) and dP issuer (R2)
    for (int s = 0; s < C::ST1; ++s) {
      mbar_init(&bar.c1_full[s], 1);
      mbar_init(&bar.c1_empty[s], 2);  // S issuer and A1 issuer
    }
    for (int s = 0; s < C::ST2; ++s) {
      mbar_init(&bar.c2_full[s], 1);
      mbar_init(&bar.c2_empty[s], KV ? 2 : 1);  // dP issuer (and A2 issuer)
    }
    mbar_init(&bar.xs_full, 1);
    mbar_init(&bar.xs_read, C::EPI_WARPS);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bar.xdp_full[b], 1);
      mbar_init(&bar.xdp_read[b], C::EPI_WARPS);
    }
    for (int q = 0; q < 4; ++q) {
      mbar_init(&bar.p_full[q], 4);
      mbar_init(&bar.ds_full[q], 4);
    }
    mbar_init(&bar.p_free, 1);
    mbar_init(&bar.ds_free, 1);
    mbar_init(&bar.acc_full, KV ? 2 : 1);
    mbar_init(&bar.acc_empty, C::EPI_WARPS);
    for (int i = 0; i < 4; ++i) mbar_init(&bar.drain[i], 1);
    ring_init(bar.ring, C::ISSUERS + C::EPI_WARPS);  // every issuer and epilogue warp reads each item
    bar.abort = 0;
    fence_mbar_init();
  }
  if (warp == kSWarp) {
    tmem_alloc(&bar.tmem_base, C::TMEM_COLS);
    tmem_relinquish();
  }
  // Zeros for the producer's bulk fill of padded dQ rows. Bulk copies need
  // 16-byte aligned addresses; the host already rejects outputs that are not,
  // and the check here keeps the rule next to the copies.
  const bool bulk_fill = C::ZBUF > 0 && fill_lengths != nullptr && (reinterpret_cast<uintptr_t>(out1) & 15u) == 0;
  // Geometry of the zero fill of the output rows no item covers (dQ, or dK
  // and dV); len_bound (Lmax) bounds the valid lengths.
  const FillGeom fill_geom{H, len_bound, L, D * (F32OUT ? 4 : 2) / 16, KV ? kKindDkdv : kKindDq, C::BM, kr};
  if (bulk_fill) {
    uint4* z = reinterpret_cast<uint4*>(smem + C::OFF_Z);
    for (int i = threadIdx.x; i < C::ZBUF / 16; i += blockDim.x) z[i] = make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();
  }
  // The plan is written by the kernel before this one in the stream. With
  // `overlap` (the dK/dV kernel of a whole-backward call) the kernel before is
  // the dQ kernel, which reads nothing this one writes and whose CTAs launch
  // this one only after their own wait for the plan: the wait moves to the end
  // (so that this grid completes after the dQ grid) and the kernel takes SMs
  // as the dQ kernel's CTAs leave them.
  if (!overlap) grid_dep_wait();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  grid_dep_launch();
  const uint32_t tmem = bar.tmem_base;
  const int count = ws[kHdrCount];
  const RowMap<PACKED> rm{H, L};

  // Descriptor bases (built once, advanced by adding (bytes >> 4): the
  // start-address field is the low 14 bits and smem stays below 256 KB).
  const uint32_t sbase = smem_u32(smem);
  constexpr uint64_t kTileC = C::TILE_C >> 4;

  if (warp < C::EPI_WARPS) {
    // ------------------------------------------------------------- epilogue
    setmaxnreg_inc<C::EPI_REGS>();
    constexpr int CPW = C::CPW, CW = C::CW, G = C::GROUPS;
    const int g = warp >> 2;                      // chunks g*CPW .. g*CPW + CPW - 1
    const int r = ((warp & 3) << 5) + lane;       // row within the item = TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) << 5) << 16;
    const uint32_t tXS = tmem + lane_off + C::TM_XS + g * CPW * CW;
    const uint32_t tXDP0 = tmem + lane_off + C::TM_XDP + g * CPW * CW;
    const uint32_t tXDP1 = tmem + lane_off + C::TM_XDP1 + g * CPW * CW;
    constexpr float scale = Scale<D>::value;
    constexpr float scale_l2e = scale * kLog2e;
    uint32_t s_ph = 0, free_ph = 0, aph = 0, xb = 0;
    uint32_t dp_ph[2] = {0, 0};
    bool ok = true;
    uint32_t ist = 0, iph = 0;
    while (ok) {
      Item item;
      if (!(ok = ring_read(bar.ring, ist, iph, &item, abort_flag, err, 220))) break;
      __syncwarp();
      ring_release(bar.ring, ist, iph, lane == 0);
      if (item.n < 0) break;
      const int n = item.n;
      const int ncols = work_cols(KV ? kKindDkdv : kKindDq, n, kr);
      const int nb = ceil_div(ncols, C::BN);
      const bool row_ok = item.blk * C::BM + r < (KV ? range_keys(n, kr) : n);  // this lane's row is a valid token
      // All 32 rows of this warp are padding (only the dQ kernel at D = 64
      // skips such work: elsewhere the extra path measured slower).
      const bool rows_dead = C::SKIP_DEAD && __all_sync(0xffffffffu, !row_ok);
      const float neg_log2n = -__log2f(static_cast<float>(n));  // bias * log2(e)
      // One column block. Padded rows are not masked (their values reach
      // only their own, discarded output rows, and they take no part in the
      // choice of sigmoid form); only the last block can hold columns past the
      // sequence, and with SPLIT_MASK it alone runs the MASKED form, which
      // sets their scores to -inf before the sigmoid.
      auto block = [&](const int j, auto masked) -> bool {
        constexpr bool MASKED = decltype(masked)::value;
        if (C::SKIP_DEAD && ((MASKED && ncols - (j * C::BN + g * CPW * CW) <= 0) || rows_dead)) {
          // No valid score in this warp's columns of the block (past the
          // sequence's end, or padded rows only): sigma' and dS are all 0.
          // The warp reads neither S nor dP and only keeps its part in the
          // hand-offs, writing zeros.
          if (!mbar_wait(&bar.xs_full, s_ph, abort_flag, err, 221)) return false;
          s_ph ^= 1;
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bar.xs_read);
          uint32_t zero[CW / 2];
#pragma unroll
          for (int e = 0; e < CW / 2; ++e) zero[e] = 0u;
          if (KV) {
            if (!mbar_wait(&bar.p_free, free_ph ^ 1, abort_flag, err, 223)) return false;
            tc_fence_after();
#pragma unroll
            for (int c = 0; c < CPW; ++c) {
              tmem_st(tmem + lane_off + C::TM_P + (g * CPW + c) * (CW / 2), zero);
              tmem_st_wait();
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(&bar.p_full[g * CPW + c]);
            }
          }
          if (!mbar_wait(&bar.xdp_full[xb], dp_ph[xb], abort_flag, err, 222)) return false;
          dp_ph[xb] ^= 1;
          uint64_t* xdp_read = &bar.xdp_read[xb];
          if (++xb == static_cast<uint32_t>(C::NXDP)) xb = 0;
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(xdp_read);
          if (!mbar_wait(&bar.ds_free, free_ph ^ 1, abort_flag, err, 224)) return false;
          free_ph ^= 1;
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < CPW; ++c) {
            tmem_st(tmem + lane_off + C::TM_DS + (g * CPW + c) * (CW / 2), zero);
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar.ds_full[g * CPW + c]);
          }
          return true;
        }
        // ---- S -> sigma'(x) = P (1 - P) kept in registers for dS, and (dK/dV)
        // bf16 P for dV, written once the previous block's dV products have
        // read the P region. Padded columns get P = sigma' = 0.
        float sp[CPW][CW];
        uint32_t pk[KV ? CPW : 1][CW / 2];
        {
          uint32_t sv[CPW][CW];
          if (!mbar_wait(&bar.xs_full, s_ph, abort_flag, err, 221)) return false;
          s_ph ^= 1;
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < CPW; ++c) tmem_ld_async(tXS + CW * c, sv[c]);
#pragma unroll
          for (int c = 0; c < CPW; ++c) tmem_ld_wait(sv[c]);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bar.xs_read);
          const int valid = ncols - (j * C::BN + g * CPW * CW);  // columns < valid are real tokens
#pragma unroll
          for (int c = 0; c < CPW; ++c) {
            if constexpr (MASKED) mask_scores(sv[c], valid - CW * c, true);
            sigmoid_n<true, CW, C::NEG_SLOPE>(sv[c], scale_l2e, neg_log2n, sp[c], row_ok);
            if (KV) {
#pragma unroll
              for (int e = 0; e < CW / 2; ++e)
                pk[KV ? c : 0][e] = pack_bf16x2(__uint_as_float(sv[c][2 * e]), __uint_as_float(sv[c][2 * e + 1]));
            }
          }
        }
        if (KV) {
          if (!mbar_wait(&bar.p_free, free_ph ^ 1, abort_flag, err, 223)) return false;
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < CPW; ++c) {
            tmem_st(tmem + lane_off + C::TM_P + (g * CPW + c) * (CW / 2), pk[KV ? c : 0]);
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar.p_full[g * CPW + c]);
          }
        }
        // ---- dP -> dS = dP P (1 - P), bf16 dS for dQ / dK: dP is copied out
        // whole, so its region is released at once.
        uint32_t dp[CPW][CW];
        const uint32_t tXDP = xb ? tXDP1 : tXDP0;
        uint64_t* xdp_read = &bar.xdp_read[xb];
        if (!mbar_wait(&bar.xdp_full[xb], dp_ph[xb], abort_flag, err, 222)) return false;
        dp_ph[xb] ^= 1;
        if (++xb == static_cast<uint32_t>(C::NXDP)) xb = 0;
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < CPW; ++c) tmem_ld_async(tXDP + CW * c, dp[c]);
#pragma unroll
        for (int c = 0; c < CPW; ++c) tmem_ld_wait(dp[c]);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(xdp_read);
        if (!mbar_wait(&bar.ds_free, free_ph ^ 1, abort_flag, err, 224)) return false;
        free_ph ^= 1;
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < CPW; ++c) {
          const uint32_t(&dpc)[CW] = dp[c];
          uint32_t dk[CW / 2];
#pragma unroll
          // -dS = dP (-sigma'): packed multiplies, except in the dK/dV kernel
          // at D = 64 (fewer registers), which measured faster with scalar
          // ones (0 %-padded 1.853 against 1.861 ms; at D = 128 packed 0.926
          // against 0.935 ms).
          for (int e = 0; e < CW / 2; ++e) {
            if constexpr (KV && D == 64) {
              dk[e] = pack_bf16x2(__uint_as_float(dpc[2 * e]) * sp[c][2 * e],
                                  __uint_as_float(dpc[2 * e + 1]) * sp[c][2 * e + 1]);
            } else {
              const float2 ds = f2_unpack(f2_mul(f2_pack(__uint_as_float(dpc[2 * e]), __uint_as_float(dpc[2 * e + 1])),
                                                 f2_pack(sp[c][2 * e], sp[c][2 * e + 1])));
              dk[e] = pack_bf16x2(ds.x, ds.y);
            }
          }
          tmem_st(tmem + lane_off + C::TM_DS + (g * CPW + c) * (CW / 2), dk);
          tmem_st_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bar.ds_full[g * CPW + c]);
        }
        return true;
      };
      if constexpr (C::SPLIT_MASK) {
        for (int j = 0; ok && j + 1 < nb; ++j) ok = block(j, std::false_type{});
        if (ok) ok = block(nb - 1, std::true_type{});
      } else {
        // One form for every block, padded rows and columns masked (the
        // block's code as one loop body, which keeps this kernel free of
        // spills).
        for (int j = 0; j < nb; ++j) {
          if (C::SKIP_DEAD && (ncols - (j * C::BN + g * CPW * CW) <= 0 || rows_dead)) {
            // No valid score in this warp's columns of the block (past the
            // sequence's end, or padded rows only): sigma' and dS are all 0.
            // The warp reads neither S nor dP and only keeps its part in the
            // hand-offs, writing zeros.
            if (!(ok = mbar_wait(&bar.xs_full, s_ph, abort_flag, err, 221))) break;
            s_ph ^= 1;
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar.xs_read);
            uint32_t zero[CW / 2];
  #pragma unroll
            for (int e = 0; e < CW / 2; ++e) zero[e] = 0u;
            if (KV) {
              if (!(ok = mbar_wait(&bar.p_free, free_ph ^ 1, abort_flag, err, 223))) break;
              tc_fence_after();
  #pragma unroll
              for (int c = 0; c < CPW; ++c) {
                tmem_st(tmem + lane_off + C::TM_P + (g * CPW + c) * (CW / 2), zero);
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&bar.p_full[g * CPW + c]);
              }
            }
            if (!(ok = mbar_wait(&bar.xdp_full[xb], dp_ph[xb], abort_flag, err, 222))) break;
            dp_ph[xb] ^= 1;
            uint64_t* xdp_read = &bar.xdp_read[xb];
            if (++xb == static_cast<uint32_t>(C::NXDP)) xb = 0;
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(xdp_read);
            if (!(ok = mbar_wait(&bar.ds_free, free_ph ^ 1, abort_flag, err, 224))) break;
            free_ph ^= 1;
            tc_fence_after();
  #pragma unroll
            for (int c = 0; c < CPW; ++c) {
              tmem_st(tmem + lane_off + C::TM_DS + (g * CPW + c) * (CW / 2), zero);
              tmem_st_wait();
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(&bar.ds_full[g * CPW + c]);
            }
            continue;
          }
          // ---- S -> sigma'(x) = P (1 - P) kept in registers for dS, and (dK/dV)
          // bf16 P for dV, written once the previous block's dV products have
          // read the P region. Padded columns get P = sigma' = 0.
          float sp[CPW][CW];
          uint32_t pk[KV ? CPW : 1][CW / 2];
          {
            uint32_t sv[CPW][CW];
            if (!(ok = mbar_wait(&bar.xs_full, s_ph, abort_flag, err, 221))) break;
            s_ph ^= 1;
            tc_fence_after();
  #pragma unroll
            for (int c = 0; c < CPW; ++c) tmem_ld_async(tXS + CW * c, sv[c]);
  #pragma unroll
            for (int c = 0; c < CPW; ++c) tmem_ld_wait(sv[c]);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar.xs_read);
            const int valid = ncols - (j * C::BN + g * CPW * CW);  // columns < valid are real tokens
  #pragma unroll
            for (int c = 0; c < CPW; ++c) {
              mask_scores(sv[c], valid - CW * c, row_ok);
              sigmoid_n<true, CW, C::NEG_SLOPE>(sv[c], scale_l2e, neg_log2n, sp[c]);
              if (KV) {
  #pragma unroll
                for (int e = 0; e < CW / 2; ++e)
                  pk[KV ? c : 0][e] = pack_bf16x2(__uint_as_float(sv[c][2 * e]), __uint_as_float(sv[c][2 * e + 1]));
              }
            }
          }
          if (KV) {
            if (!(ok = mbar_wait(&bar.p_free, free_ph ^ 1, abort_flag, err, 223))) break;
            tc_fence_after();
  #pragma unroll
            for (int c = 0; c < CPW; ++c) {
              tmem_st(tmem + lane_off + C::TM_P + (g * CPW + c) * (CW / 2), pk[KV ? c : 0]);
              tmem_st_wait();
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(&bar.p_full[g * CPW + c]);
            }
          }
          // ---- dP -> dS = dP P (1 - P), bf16 dS for dQ / dK: dP is copied out
          // whole, so its region is released at once.
          uint32_t dp[CPW][CW];
          const uint32_t tXDP = xb ? tXDP1 : tXDP0;
          uint64_t* xdp_read = &bar.xdp_read[xb];
          if (!(ok = mbar_wait(&bar.xdp_full[xb], dp_ph[xb], abort_flag, err, 222))) break;
          dp_ph[xb] ^= 1;
          if (++xb == static_cast<uint32_t>(C::NXDP)) xb = 0;
          tc_fence_after();
  #pragma unroll
          for (int c = 0; c < CPW; ++c) tmem_ld_async(tXDP + CW * c, dp[c]);
  #pragma unroll
          for (int c = 0; c < CPW; ++c) tmem_ld_wait(dp[c]);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(xdp_read);
          if (!(ok = mbar_wait(&bar.ds_free, free_ph ^ 1, abort_flag, err, 224))) break;
          free_ph ^= 1;
          tc_fence_after();
  #pragma unroll
          for (int c = 0; c < CPW; ++c) {
            const uint32_t(&dpc)[CW] = dp[c];
            uint32_t dk[CW / 2];
  #pragma unroll
            // -dS = dP (-sigma'): packed multiplies, except in the dK/dV kernel
            // at D = 64 (fewer registers), which measured faster with scalar
            // ones (0 %-padded 1.853 against 1.861 ms; at D = 128 packed 0.926
            // against 0.935 ms).
            for (int e = 0; e < CW / 2; ++e) {
              if constexpr (KV && D == 64) {
                dk[e] = pack_bf16x2(__uint_as_float(dpc[2 * e]) * sp[c][2 * e],
                                    __uint_as_float(dpc[2 * e + 1]) * sp[c][2 * e + 1]);
              } else {
                const float2 ds = f2_unpack(f2_mul(f2_pack(__uint_as_float(dpc[2 * e]), __uint_as_float(dpc[2 * e + 1])),
                                                   f2_pack(sp[c][2 * e], sp[c][2 * e + 1])));
                dk[e] = pack_bf16x2(ds.x, ds.y);
              }
            }
            tmem_st(tmem + lane_off + C::TM_DS + (g * CPW + c) * (CW / 2), dk);
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar.ds_full[g * CPW + c]);
          }
        }
      }
      if (!ok) break;
      if (!(ok = mbar_wait(&bar.acc_full, aph, abort_flag, err, 225))) break;
      aph ^= 1;
      tc_fence_after();
      const int row = item.blk * C::BM + r;
      const bool in_range = rm.writes(row, n);
      const bool valid_row = row < (KV ? range_keys(n, kr) : n);
      const size_t row_off = rm.offset(item, PACKED ? item.bh % H : 0, row, D);
      // Chunks of RW accumulator columns (32, or 16 where the column groups
      // outnumber the 32-column chunks): A1 (-> out1, times scale), then A2
      // (-> out2) for dK/dV; column group g takes chunks g, g + G, ...
      // Each chunk is copied out and packed to bf16 at once, so the
      // accumulators are released before the (slower) global stores.
      constexpr int kCols = (KV ? 2 : 1) * D;
      constexpr int RW = kCols / G >= 32 ? 32 : 16;
      constexpr int kChunks = kCols / RW;
      constexpr int kPer = kChunks / G;
      static_assert(kPer * G == kChunks, "accumulator chunks");
      // bf16 pairs, or (F32OUT) the fp32 values themselves
      constexpr int kWords = F32OUT ? RW : RW / 2;
      uint32_t packed[kPer][kWords];
#pragma unroll
      for (int i = 0; i < kPer; ++i) {
        const int c = g + G * i;
        const bool second = c >= D / RW;
        const int col = (second ? c - D / RW : c) * RW;
        // with NEG_SLOPE the accumulators hold -dS K (dQ), or -dS^T Q and
        // -P^T dO (dK, dV): they take -scale and -1
        const float mul = (second ? 1.0f : scale) * (C::NEG_SLOPE ? -1.0f : 1.0f) * (valid_row ? 1.0f : 0.0f);
        uint32_t v[RW];
        tmem_ld_async(tmem + lane_off + (second ? C::TM_A2 : C::TM_A1) + col, v);
        tmem_ld_wait(v);
        if constexpr (F32OUT) {
#pragma unroll
          for (int e = 0; e < RW; ++e) packed[i][e] = valid_row ? __float_as_uint(__uint_as_float(v[e]) * mul) : 0u;
        } else {
#pragma unroll
          for (int e = 0; e < RW / 2; ++e)
            packed[i][e] = valid_row ? pack_bf16x2(__uint_as_float(v[2 * e]) * mul, __uint_as_float(v[2 * e + 1]) * mul)
                                     : 0u;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar.acc_empty);
      if (in_range) {  // rows past the valid ones get zeros
#pragma unroll
        for (int i = 0; i < kPer; ++i) {
          const int c = g + G * i;
          const bool second = c >= D / RW;
          const int col = (second ? c - D / RW : c) * RW;
          void* out = second ? out2 : out1;
          const size_t off = (row_off + col) * (F32OUT ? 4 : 2);
          store_words(static_cast<uint8_t*>(out) + off, packed[i]);
        }
      }
    }
  } else {
    // The producer, the issuers and the idle warps (one warpgroup pair) hand
    // registers to the epilogue.
    setmaxnreg_dec<C::OTHER_REGS>();
    if (warp == kProducerWarp) {
      // ------------------------------------------------------------- producer
      if (lane == 0) {
        tma_prefetch_desc(&tm_r1);
        tma_prefetch_desc(&tm_r2);
        tma_prefetch_desc(&tm_c1);
        tma_prefetch_desc(&tm_c2);
        uint32_t s1 = 0, p1 = 0, s2 = 0, p2 = 0, rph = 0;
        int c1_last[C::ST1], c2_last[C::ST2], r_last = -1;
        for (int s = 0; s < C::ST1; ++s) c1_last[s] = -1;
        for (int s = 0; s < C::ST2; ++s) c2_last[s] = -1;
        bool ok = true;
        uint32_t ist = 0, iph = 0;
        int claimed = -1;
        // Bulk zero fill: one unit per work item, claimed one item ahead so
        // that the atomic's latency is not waited for.
        const long long fill_units = bulk_fill ? static_cast<long long>(B) * H * fill_parts : 0;
        int fill_u = -1;
        auto issue_fill = [&]() {
          if constexpr (C::ZBUF > 0) {
            if (fill_u >= 0 && fill_u < fill_units) {
              const FillRange f = zero_fill_range(fill_lengths, fill_geom, fill_parts, fill_u);
              uint8_t* g = reinterpret_cast<uint8_t*>(out1) + f.base * 16;
              constexpr long long kPiece = C::ZBUF / 16;  // 16-byte chunks per bulk copy
              for (long long c = f.begin; c < f.end; c += kPiece)
                bulk_store(g + c * 16, sbase + C::OFF_Z, static_cast<uint32_t>(min(kPiece, f.end - c) * 16));
              bulk_commit();
            }
          }
        };
        while (ok) {
          const Item item = next_item(ws, claimed, count);
          if (!(ok = ring_publish(bar.ring, ist, iph, item, abort_flag, err, 200))) break;
          if (item.n < 0) break;
          const int n = item.n;
          const int hd = PACKED ? item.bh % H : 0;
          const int nb = ceil_div(work_cols(KV ? kKindDkdv : kKindDq, n, kr), C::BN);
          if (fill_units > 0 && fill_u < fill_units) {
            issue_fill();
            fill_u = atomicAdd(ws + kHdrFill, 1);
          }
          if (!(ok = mbar_wait(&bar.r_empty, rph ^ 1, abort_flag, err, 201))) break;
          mbar_arrive_expect_tx(&bar.r_full, 2 * C::TILE_R);
          for (int c = 0; c < D / 64; ++c) {
            const int ry = rm.y(item, hd, item.blk * C::BM), rz = rm.z(item, item.blk * C::BM);
            tma_load_3d(smem + C::OFF_R1 + c * C::BOX_R, &tm_r1, &bar.r_full, c * 64, ry, rz);
            tma_load_3d(smem + C::OFF_R2 + c * C::BOX_R, &tm_r2, &bar.r_full, c * 64, ry, rz);
          }
          r_last = static_cast<int>(rph);
          rph ^= 1;
          for (int j = 0; j < nb; ++j) {
            // Claim the CTA's next item two column blocks before this one ends.
            if (j == max(0, nb - 2)) claimed = atomicAdd(ws + kHdrNext, 1);
            if (!(ok = mbar_wait(&bar.c1_empty[s1], p1 ^ 1, abort_flag, err, 202))) break;
            mbar_arrive_expect_tx(&bar.c1_full[s1], C::TILE_C);
            for (int c = 0; c < D / 64; ++c)
              tma_load_3d(smem + C::OFF_C1 + s1 * C::TILE_C + c * C::BOX_C, &tm_c1, &bar.c1_full[s1], c * 64,
                          rm.y(item, hd, j * C::BN), rm.z(item, j * C::BN));
            c1_last[s1] = static_cast<int>(p1);
            if (++s1 == C::ST1) { s1 = 0; p1 ^= 1; }
            if (!(ok = mbar_wait(&bar.c2_empty[s2], p2 ^ 1, abort_flag, err, 203))) break;
            mbar_arrive_expect_tx(&bar.c2_full[s2], C::TILE_C);
            for (int c = 0; c < D / 64; ++c)
              tma_load_3d(smem + C::OFF_C2 + s2 * C::TILE_C + c * C::BOX_C, &tm_c2, &bar.c2_full[s2], c * 64,
                          rm.y(item, hd, j * C::BN), rm.z(item, j * C::BN));
            c2_last[s2] = static_cast<int>(p2);
            if (++s2 == C::ST2) { s2 = 0; p2 ^= 1; }
          }
        }
        // The last unit claimed, then every bulk copy must have landed before
        // the shared-memory zeros go away with the CTA.
        if (fill_units > 0) {
          issue_fill();
          bulk_wait_all();
        }
        if (!ok) {  // aborting: let the copies in flight land before the CTA exits
          int never = 0;
          volatile int* no_abort = &never;
          for (int s = 0; s < C::ST1; ++s)
            if (c1_last[s] >= 0) mbar_wait(&bar.c1_full[s], c1_last[s], no_abort, nullptr, 0);
          for (int s = 0; s < C::ST2; ++s)
            if (c2_last[s] >= 0) mbar_wait(&bar.c2_full[s], c2_last[s], no_abort, nullptr, 0);
          if (r_last >= 0) mbar_wait(&bar.r_full, r_last, no_abort, nullptr, 0);
        }
      }
    } else if (warp == kSWarp || warp == kDPWarp) {
      // ------------------------------------------ issuers of S = R1 C1^T, dP = R2 C2^T
      if (lane == 0) {
        const bool is_dp = (warp == kDPWarp);
        constexpr uint32_t idesc_x = idesc_bf16_f32(128, C::BN, false, false);
        const uint64_t d_r = smem_desc_sw128(sbase + (is_dp ? C::OFF_R2 : C::OFF_R1), 16, 1024);
        const uint64_t d_c = smem_desc_sw128(sbase + (is_dp ? C::OFF_C2 : C::OFF_C1), 16, 1024);
        const int nbuf = is_dp ? C::NXDP : 1;     // regions this issuer rotates through
        const int slots = is_dp ? C::ST2 : C::ST1;
        uint64_t* cfull = is_dp ? bar.c2_full : bar.c1_full;
        uint64_t* cempty = is_dp ? bar.c2_empty : bar.c1_empty;
        uint32_t st = 0, cph = 0, rph = 0, xb = 0;
        uint32_t read_ph[2] = {0, 0};
        bool ok = true;
        uint32_t ist = 0, iph = 0;
        while (ok) {
          Item item;
          if (!(ok = ring_read(bar.ring, ist, iph, &item, abort_flag, err, 210))) break;
          ring_release(bar.ring, ist, iph, true);
          if (item.n < 0) break;
          const int n = item.n;
          const int nb = ceil_div(work_cols(KV ? kKindDkdv : kKindDq, n, kr), C::BN);
          if (!(ok = mbar_wait(&bar.r_full, rph, abort_flag, err, 211))) break;
          rph ^= 1;
          for (int j = 0; j < nb; ++j) {
            if (!(ok = mbar_wait(&cfull[st], cph, abort_flag, err, 212))) break;
            // The region is free once the epilogue has copied out the block that
            // last used it (block j-1, or j-2 with two dP regions).
            uint64_t* xread = is_dp ? &bar.xdp_read[xb] : &bar.xs_read;
            uint64_t* xfull = is_dp ? &bar.xdp_full[xb] : &bar.xs_full;
            const uint32_t d_tmem = tmem + (is_dp ? (xb ? C::TM_XDP1 : C::TM_XDP) : C::TM_XS);
            if (!(ok = mbar_wait(xread, read_ph[xb] ^ 1, abort_flag, err, 213))) break;
            read_ph[xb] ^= 1;
            tc_fence_after();
            const uint64_t b0 = d_c + st * kTileC;
  #pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {  // K = D in steps of 16
              const uint64_t a_off = ((kk >> 2) * C::BOX_R + (kk & 3) * 32) >> 4;
              const uint64_t b_off = ((kk >> 2) * C::BOX_C + (kk & 3) * 32) >> 4;
              mma_ss(d_tmem, d_r + a_off, b0 + b_off, idesc_x, kk > 0 ? 1u : 0u);
            }
            mma_commit(xfull);
            mma_commit(&cempty[st]);
            if (++st == slots) { st = 0; cph ^= 1; }
            if (++xb == static_cast<uint32_t>(nbuf)) xb = 0;
            if (j + 1 == nb) mma_commit(&bar.r_empty);
          }
        }
        int never = 0;
        mma_commit(&bar.drain[is_dp ? 1 : 0]);
        mbar_wait(&bar.drain[is_dp ? 1 : 0], 0, &never, err, 219);
      }
    } else if (warp == kA1Warp || warp == kA2Warp) {
      // -------------------------- issuers of A1 += dS C1 and (dK/dV) A2 += P C2
      if (lane == 0) {
        const bool second = (warp == kA2Warp);
        constexpr uint32_t idesc_acc = idesc_bf16_f32(128, D, false, true);
        // MN-major view of the C1 (A1) or C2 (A2) ring: rows = the K dimension,
        // the two 64-column halves of D BOX_C bytes apart.
        const uint64_t d_cmn = smem_desc_sw128(sbase + (second ? C::OFF_C2 : C::OFF_C1), C::BOX_C, 1024);
        const int slots = second ? C::ST2 : C::ST1;
        uint64_t* cfull = second ? bar.c2_full : bar.c1_full;
        uint64_t* cempty = second ? bar.c2_empty : bar.c1_empty;
        const uint32_t tm_acc = tmem + (second ? C::TM_A2 : C::TM_A1);
        const uint32_t tm_a = tmem + (second ? C::TM_P : C::TM_DS);
        uint64_t* full = second ? bar.p_full : bar.ds_full;
        uint64_t* freed = second ? &bar.p_free : &bar.ds_free;
        uint32_t st = 0, cph = 0, aph = 0;
        uint32_t fph[4] = {0, 0, 0, 0};
        bool ok = true;
        uint32_t ist = 0, iph = 0;
        while (ok) {
          Item item;
          if (!(ok = ring_read(bar.ring, ist, iph, &item, abort_flag, err, 210))) break;
          ring_release(bar.ring, ist, iph, true);
          if (item.n < 0) break;
          const int n = item.n;
          const int nb = ceil_div(work_cols(KV ? kKindDkdv : kKindDq, n, kr), C::BN);
          for (int j = 0; ok && j < nb; ++j) {
            if (!(ok = mbar_wait(&cfull[st], cph, abort_flag, err, 231))) break;
            const uint64_t b0 = d_cmn + st * kTileC;
            for (int q = 0; q < C::NCH; ++q) {
              if (!(ok = mbar_wait(&full[q], fph[q], abort_flag, err, 232))) break;
              fph[q] ^= 1;
              const bool first = (j == 0 && q == 0);
              if (first) {
                if (!(ok = mbar_wait(&bar.acc_empty, aph ^ 1, abort_flag, err, 233))) break;
                aph ^= 1;
              }
              tc_fence_after();
              // K = the chunk's CW columns in K=16 steps; the chunk's bf16
              // values sit in CW/2 TMEM columns (two per column).
  #pragma unroll
              for (int kk = 0; kk < C::CW / 16; ++kk)
                mma_ts(tm_acc, tm_a + q * (C::CW / 2) + kk * 8, b0 + ((q * C::CW * 128 + kk * 2048) >> 4),
                       idesc_acc, (first && kk == 0) ? 0u : 1u);
            }
            if (!ok) break;
            mma_commit(freed);
            mma_commit(&cempty[st]);
            if (++st == slots) { st = 0; cph ^= 1; }
          }
          if (!ok) break;
          mma_commit(&bar.acc_full);
        }
        int never = 0;
        mma_commit(&bar.drain[second ? 3 : 2]);
        mbar_wait(&bar.drain[second ? 3 : 2], 0, &never, err, 239);
      }
    }
  }

  // Padded inputs: the output rows no item covers are zeroed by the warps
  // without a role from the start (they come straight here) and by every other
  // warp once its role is done, claiming fill units from the workspace counter
  // that the dQ kernel's producer also takes units from for its bulk copies.
  if (fill_lengths != nullptr) {
    const long long units = static_cast<long long>(B) * H * fill_parts;
    while (true) {
      int u = 0;
      if (lane == 0) u = atomicAdd(ws + kHdrFill, 1);
      u = __shfl_sync(0xffffffffu, u, 0);
      if (u >= units) break;
      const FillRange f = zero_fill_range(fill_lengths, fill_geom, fill_parts, u);
      zero_fill_range_warp(f, lane, out1);
      if (KV) zero_fill_range_warp(f, lane, out2);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kSWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
  if (overlap) grid_dep_wait();
}

template <int D, bool KV, bool PACKED, bool F32OUT>
cudaError_t launch_bwd_impl(const CUtensorMap& r1, const CUtensorMap& r2, const CUtensorMap& c1,
                            const CUtensorMap& c2, void* out1, void* out2, int* ws, int B, int H, int L, KeyRange kr,
                            int num_sms, const int* fill_lengths, int len_bound, cudaStream_t stream,
                            const BwdLink& link) {
  using C = BwdCfg<D, KV>;
  static PerDeviceOnce attr;
  const cudaError_t e = attr.run([] {
    cudaError_t r = cudaFuncSetAttribute(bwd_kernel<D, KV, PACKED, F32OUT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_ALLOC);
    if (r != cudaSuccess) return r;
    // The setmaxnreg split draws on the registers the CTA is launched with:
    // refuse to launch if the compiler allocated fewer than the split needs
    // (the epilogue's increase would otherwise wait for ever).
    cudaFuncAttributes fa;
    r = cudaFuncGetAttributes(&fa, bwd_kernel<D, KV, PACKED, F32OUT>);
    if (r != cudaSuccess) return r;
    const long long need = (static_cast<long long>(C::EPI_REGS) * C::EPI_WARPS +
                            static_cast<long long>(C::OTHER_REGS) * (C::WARPS - C::EPI_WARPS)) * 32;
    return static_cast<long long>(fa.numRegs) * C::THREADS >= need ? cudaSuccess : cudaErrorLaunchOutOfResources;
  });
  if (e != cudaSuccess) return e;
  const long long max_items = static_cast<long long>(B) * H * ceil_div(L, kBwdItemRows);
  const int grid = static_cast<int>(std::min<long long>(num_sms, max_items));
  const int parts = zero_fill_parts(static_cast<long long>(B) * H, num_sms);
  return launch_programmatic(bwd_kernel<D, KV, PACKED, F32OUT>, dim3(grid), dim3(C::THREADS), C::SMEM_ALLOC, stream,
                             r1, r2, c1, c2, out1, out2, ws, H, L, kr, fill_lengths, B, len_bound, parts,
                             link.err != nullptr ? link.err : ws, link.overlap ? 1 : 0);
}

// fill_lengths: the padded layout's lengths, so that the kernel zeroes the
// output rows no item covers itself (nullptr for the packed layout, whose
// calls write only the rows of the sequences). kr: the keys the call covers
// ({0, L} for whole sequences); f32out: dQ as the fp32 partial sum over them.
cudaError_t launch_bwd_dq(int d, bool packed, bool f32out, const CUtensorMap& tq, const CUtensorMap& tdo,
                          const CUtensorMap& tk, const CUtensorMap& tv, void* dq, int* ws, int B, int H, int L,
                          KeyRange kr, int num_sms, const int* fill_lengths, cudaStream_t stream,
                          const BwdLink& link) {
  if (packed) {
    if (d == 64)
      return launch_bwd_impl<64, false, true, false>(tq, tdo, tk, tv, dq, nullptr, ws, B, H, L, kr, num_sms, nullptr,
                                                     L, stream, link);
    return launch_bwd_impl<128, false, true, false>(tq, tdo, tk, tv, dq, nullptr, ws, B, H, L, kr, num_sms, nullptr,
                                                    L, stream, link);
  }
  if (f32out) {
    if (d == 64)
      return launch_bwd_impl<64, false, false, true>(tq, tdo, tk, tv, dq, nullptr, ws, B, H, L, kr, num_sms,
                                                     fill_lengths, L, stream, link);
    return launch_bwd_impl<128, false, false, true>(tq, tdo, tk, tv, dq, nullptr, ws, B, H, L, kr, num_sms,
                                                    fill_lengths, L, stream, link);
  }
  if (d == 64)
    return launch_bwd_impl<64, false, false, false>(tq, tdo, tk, tv, dq, nullptr, ws, B, H, L, kr, num_sms,
                                                    fill_lengths, L, stream, link);
  return launch_bwd_impl<128, false, false, false>(tq, tdo, tk, tv, dq, nullptr, ws, B, H, L, kr, num_sms,
                                                   fill_lengths, L, stream, link);
}

// out_rows: rows per (b, h) slice of dK and dV (Lmax, or kr.count for a key
// range, whose K and V maps hold only the range's keys); Lmax bounds the valid
// lengths.
cudaError_t launch_bwd_dkdv(int d, bool packed, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tq,
                            const CUtensorMap& tdo, void* dk, void* dv, int* ws, int B, int H, int out_rows, int Lmax,
                            KeyRange kr, int num_sms, const int* fill_lengths, cudaStream_t stream,
                            const BwdLink& link) {
  if (packed) {
    if (d == 64)
      return launch_bwd_impl<64, true, true, false>(tk, tv, tq, tdo, dk, dv, ws, B, H, out_rows, kr, num_sms, nullptr,
                                                    Lmax, stream, link);
    return launch_bwd_impl<128, true, true, false>(tk, tv, tq, tdo, dk, dv, ws, B, H, out_rows, kr, num_sms, nullptr,
                                                   Lmax, stream, link);
  }
  if (d == 64)
    return launch_bwd_impl<64, true, false, false>(tk, tv, tq, tdo, dk, dv, ws, B, H, out_rows, kr, num_sms,
                                                   fill_lengths, Lmax, stream, link);
  return launch_bwd_impl<128, true, false, false>(tk, tv, tq, tdo, dk, dv, ws, B, H, out_rows, kr, num_sms,
                                                  fill_lengths, Lmax, stream, link);
}

}  // namespace sigattn
