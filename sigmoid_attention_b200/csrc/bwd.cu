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
// Each 128-column block is processed as two 64-column halves g = 0, 1, one
// per epilogue warpgroup, so that the tensor core computes one half while the
// other half's epilogue runs:
//   S_g  = R1 C1[g]^T, dP_g = R2 C2[g]^T       (tcgen05.mma, both operands in smem)
//   epilogue g: P = sigma(S*scale + b) (0 for padded columns), dS = dP P (1-P),
//               written back as bf16 into the first 32 columns of S_g / dP_g
//   A1 += dS_g C1[g], A2 += P_g C2[g]          (tcgen05.mma with A read from TMEM)
// Warps: 0-3 epilogue half 0, 4-7 epilogue half 1, 8 TMA producer, 9 MMA.
// TMEM: S_g at 64g, dP_g at 128 + 64g, A1 at 256, A2 at 256 + D.
#include "common.cuh"

namespace sigattn {

template <int D, bool KV>
struct BwdCfg {
  static constexpr int BM = kBwdItemRows;   // 128 rows per item
  static constexpr int BN = kColBlock;      // 128 columns per block
  static constexpr int ST = (D == 128) ? 2 : 3;
  static constexpr int BOX_BYTES = 128 * 64 * 2;
  static constexpr int TILE_BYTES = 128 * D * 2;
  static constexpr int OFF_R1 = 0;
  static constexpr int OFF_R2 = TILE_BYTES;
  static constexpr int OFF_C = 2 * TILE_BYTES;  // stage s: C1 at OFF_C + 2s*TILE, C2 right after
  static constexpr int SMEM_BYTES = OFF_C + ST * 2 * TILE_BYTES;
  static constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;
  static constexpr int TM_S = 0;
  static constexpr int TM_DP = 128;
  static constexpr int TM_A1 = 256;
  static constexpr int TM_A2 = 256 + D;
  static constexpr int TMEM_COLS = 512;
  static constexpr int THREADS = 320;
};

template <int ST>
struct BwdBarriers {
  uint64_t r_full, r_empty;
  uint64_t c_full[ST], c_empty[ST];
  uint64_t s_full[2], p_full[2];
  uint64_t acc_full, acc_empty;
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

// Convert 32 fp32 accumulator values (times `mul`) to bf16 and store them.
__device__ __forceinline__ void store_row32(__nv_bfloat16* dst, const uint32_t (&v)[32], float mul) {
  uint4* p = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    p[q] = make_uint4(pack_bf16x2(__uint_as_float(v[8 * q + 0]) * mul, __uint_as_float(v[8 * q + 1]) * mul),
                      pack_bf16x2(__uint_as_float(v[8 * q + 2]) * mul, __uint_as_float(v[8 * q + 3]) * mul),
                      pack_bf16x2(__uint_as_float(v[8 * q + 4]) * mul, __uint_as_float(v[8 * q + 5]) * mul),
                      pack_bf16x2(__uint_as_float(v[8 * q + 6]) * mul, __uint_as_float(v[8 * q + 7]) * mul));
  }
}

__device__ __forceinline__ void store_zero32(__nv_bfloat16* dst) {
  uint4* p = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int q = 0; q < 4; ++q) p[q] = make_uint4(0, 0, 0, 0);
}

template <int D, bool KV>
__global__ void __launch_bounds__(320, 1)
    bwd_kernel(const __grid_constant__ CUtensorMap tm_r1, const __grid_constant__ CUtensorMap tm_r2,
               const __grid_constant__ CUtensorMap tm_c1, const __grid_constant__ CUtensorMap tm_c2,
               __nv_bfloat16* __restrict__ out1, __nv_bfloat16* __restrict__ out2,
               const int* __restrict__ lengths, int* __restrict__ ws, int H, int L) {
  using C = BwdCfg<D, KV>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ BwdBarriers<C::ST> bar;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  volatile int* abort_flag = &bar.abort;

  if (threadIdx.x == 0) {
    mbar_init(&bar.r_full, 1);
    mbar_init(&bar.r_empty, 1);
    for (int s = 0; s < C::ST; ++s) { mbar_init(&bar.c_full[s], 1); mbar_init(&bar.c_empty[s], 1); }
    for (int g = 0; g < 2; ++g) { mbar_init(&bar.s_full[g], 1); mbar_init(&bar.p_full[g], 4); }
    mbar_init(&bar.acc_full, 1);
    mbar_init(&bar.acc_empty, 8);
    mbar_init(&bar.drain, 1);
    bar.abort = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(&bar.tmem_base, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar.tmem_base;
  const int count = ws[kHdrCount];

  if (warp == 8) {
    // ------------------------------------------------------------- producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_r1);
      tma_prefetch_desc(&tm_r2);
      tma_prefetch_desc(&tm_c1);
      tma_prefetch_desc(&tm_c2);
      uint32_t st = 0, cph = 0, rph = 0;
      int c_last[C::ST], r_last = -1;
      for (int s = 0; s < C::ST; ++s) c_last[s] = -1;
      bool ok = true;
      for (int it = blockIdx.x; ok && it < count; it += gridDim.x) {
        const Item item = load_item(ws, it);
        const int n = load_len(lengths, item.bh / H, L);
        const int nb = ceil_div(n, C::BN);
        if (!(ok = mbar_wait(&bar.r_empty, rph ^ 1, abort_flag, ws, 201))) break;
        mbar_arrive_expect_tx(&bar.r_full, 2 * C::TILE_BYTES);
        for (int c = 0; c < D / 64; ++c) {
          tma_load_3d(smem + C::OFF_R1 + c * C::BOX_BYTES, &tm_r1, &bar.r_full, c * 64, item.blk * C::BM, item.bh);
          tma_load_3d(smem + C::OFF_R2 + c * C::BOX_BYTES, &tm_r2, &bar.r_full, c * 64, item.blk * C::BM, item.bh);
        }
        r_last = static_cast<int>(rph);
        rph ^= 1;
        for (int j = 0; j < nb; ++j) {
          if (!(ok = mbar_wait(&bar.c_empty[st], cph ^ 1, abort_flag, ws, 202))) break;
          mbar_arrive_expect_tx(&bar.c_full[st], 2 * C::TILE_BYTES);
          uint8_t* c1 = smem + C::OFF_C + st * 2 * C::TILE_BYTES;
          uint8_t* c2 = c1 + C::TILE_BYTES;
          for (int c = 0; c < D / 64; ++c) {
            tma_load_3d(c1 + c * C::BOX_BYTES, &tm_c1, &bar.c_full[st], c * 64, j * C::BN, item.bh);
            tma_load_3d(c2 + c * C::BOX_BYTES, &tm_c2, &bar.c_full[st], c * 64, j * C::BN, item.bh);
          }
          c_last[st] = static_cast<int>(cph);
          if (++st == C::ST) { st = 0; cph ^= 1; }
        }
      }
      if (!ok) {  // aborting: let the copies in flight land before the CTA exits
        int never = 0;
        volatile int* no_abort = &never;
        for (int s = 0; s < C::ST; ++s)
          if (c_last[s] >= 0) mbar_wait(&bar.c_full[s], c_last[s], no_abort, nullptr, 0);
        if (r_last >= 0) mbar_wait(&bar.r_full, r_last, no_abort, nullptr, 0);
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_sd = idesc_bf16_f32(128, 64, false, false);
      constexpr uint32_t idesc_acc = idesc_bf16_f32(128, D, false, true);
      const uint32_t base = smem_u32(smem);
      uint32_t st = 0, cph = 0, rph = 0, aph = 0;
      uint32_t pph[2] = {0, 0};
      bool ok = true;

      // S_g = R1 C1[g]^T and dP_g = R2 C2[g]^T for the 64 columns of half g.
      auto issue_sdp = [&](int g, uint32_t s) {
        const uint32_t c1 = base + C::OFF_C + s * 2 * C::TILE_BYTES + g * 64 * 128;
        const uint32_t c2 = c1 + C::TILE_BYTES;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::BOX_BYTES + (kk & 3) * 32;
          mma_ss(tmem + C::TM_S + g * 64, smem_desc_sw128(base + C::OFF_R1 + off, 16, 1024),
                 smem_desc_sw128(c1 + off, 16, 1024), idesc_sd, kk > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::BOX_BYTES + (kk & 3) * 32;
          mma_ss(tmem + C::TM_DP + g * 64, smem_desc_sw128(base + C::OFF_R2 + off, 16, 1024),
                 smem_desc_sw128(c2 + off, 16, 1024), idesc_sd, kk > 0 ? 1u : 0u);
        }
      };
      // A1 += dS_g C1[g] (and A2 += P_g C2[g]); K = the 64 columns of half g.
      auto issue_acc = [&](int g, uint32_t s, bool acc) {
        const uint32_t c1 = base + C::OFF_C + s * 2 * C::TILE_BYTES + g * 64 * 128;
        const uint32_t c2 = c1 + C::TILE_BYTES;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          mma_ts(tmem + C::TM_A1, tmem + C::TM_DP + g * 64 + kk * 8,
                 smem_desc_sw128(c1 + kk * 2048, C::BOX_BYTES, 1024), idesc_acc, (acc || kk > 0) ? 1u : 0u);
          if (KV)
            mma_ts(tmem + C::TM_A2, tmem + C::TM_S + g * 64 + kk * 8,
                   smem_desc_sw128(c2 + kk * 2048, C::BOX_BYTES, 1024), idesc_acc, (acc || kk > 0) ? 1u : 0u);
        }
      };

      for (int it = blockIdx.x; ok && it < count; it += gridDim.x) {
        const Item item = load_item(ws, it);
        const int n = load_len(lengths, item.bh / H, L);
        const int nb = ceil_div(n, C::BN);
        if (!(ok = mbar_wait(&bar.r_full, rph, abort_flag, ws, 211))) break;
        rph ^= 1;
        if (!(ok = mbar_wait(&bar.c_full[st], cph, abort_flag, ws, 212))) break;
        tc_fence_after();
        for (int g = 0; g < 2; ++g) {
          issue_sdp(g, st);
          mma_commit(&bar.s_full[g]);
        }
        if (nb == 1) mma_commit(&bar.r_empty);
        for (int j = 0; ok && j < nb; ++j) {
          const bool has_next = (j + 1 < nb);
          const uint32_t cur = st;
          uint32_t nxt = st + 1, nph = cph;
          if (nxt == C::ST) { nxt = 0; nph ^= 1; }
          for (int g = 0; g < 2; ++g) {
            if (!(ok = mbar_wait(&bar.p_full[g], pph[g], abort_flag, ws, 213))) break;
            pph[g] ^= 1;
            if (j == 0 && g == 0) {
              if (!(ok = mbar_wait(&bar.acc_empty, aph ^ 1, abort_flag, ws, 214))) break;
              aph ^= 1;
            }
            tc_fence_after();
            issue_acc(g, cur, !(j == 0 && g == 0));
            if (has_next) {
              if (g == 0) {
                if (!(ok = mbar_wait(&bar.c_full[nxt], nph, abort_flag, ws, 215))) break;
                tc_fence_after();
              }
              issue_sdp(g, nxt);
              mma_commit(&bar.s_full[g]);
            }
          }
          if (!ok) break;
          if (has_next && j + 2 == nb) mma_commit(&bar.r_empty);
          mma_commit(&bar.c_empty[cur]);
          st = nxt;
          cph = nph;
        }
        if (!ok) break;
        mma_commit(&bar.acc_full);
      }
      int never = 0;
      mma_commit(&bar.drain);
      mbar_wait(&bar.drain, 0, &never, ws, 219);
    }
  } else {
    // ------------------------------------------------------------- epilogue
    const int g = warp >> 2;                      // column half of this warpgroup
    const int r = ((warp & 3) << 5) + lane;       // row within the item = TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) << 5) << 16;
    const uint32_t tS = tmem + lane_off + C::TM_S + g * 64;
    const uint32_t tDP = tmem + lane_off + C::TM_DP + g * 64;
    constexpr float scale = Scale<D>::value;
    constexpr float half_scale = 0.5f * scale;
    uint32_t sph = 0, aph = 0;
    bool ok = true;
    for (int it = blockIdx.x; ok && it < count; it += gridDim.x) {
      const Item item = load_item(ws, it);
      const int n = load_len(lengths, item.bh / H, L);
      const int nb = ceil_div(n, C::BN);
      const float half_bias = -0.5f * __logf(static_cast<float>(n));
      for (int j = 0; j < nb; ++j) {
        if (!(ok = mbar_wait(&bar.s_full[g], sph, abort_flag, ws, 221))) break;
        sph ^= 1;
        tc_fence_after();
        const int valid = n - (j * C::BN + g * 64);  // columns < valid are real tokens
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t s[32], dp[32];
          tmem_ld32x2(tS + c * 32, tDP + c * 32, s, dp);
          uint32_t pk_p[16], pk_ds[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            float p0 = sigmoid_from_score(__uint_as_float(s[2 * e]), half_scale, half_bias);
            float p1 = sigmoid_from_score(__uint_as_float(s[2 * e + 1]), half_scale, half_bias);
            if (valid < 64) {
              const int col = c * 32 + 2 * e;
              p0 = (col < valid) ? p0 : 0.f;
              p1 = (col + 1 < valid) ? p1 : 0.f;
            }
            const float ds0 = __uint_as_float(dp[2 * e]) * (p0 - p0 * p0);
            const float ds1 = __uint_as_float(dp[2 * e + 1]) * (p1 - p1 * p1);
            pk_p[e] = pack_bf16x2(p0, p1);
            pk_ds[e] = pack_bf16x2(ds0, ds1);
          }
          // bf16 results for columns [32c, 32c+32) go to TMEM columns
          // [16c, 16c+16) of the same region: already read by this thread.
          if (KV) tmem_st16(tS + c * 16, pk_p);
          tmem_st16(tDP + c * 16, pk_ds);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar.p_full[g]);
      }
      if (!ok) break;
      if (!(ok = mbar_wait(&bar.acc_full, aph, abort_flag, ws, 222))) break;
      aph ^= 1;
      tc_fence_after();
      const int row = item.blk * C::BM + r;
      const bool in_range = row < L;
      const bool valid_row = row < n;
      const size_t row_off = (static_cast<size_t>(item.bh) * L + row) * D;
      if (!KV) {
        // dQ: warpgroup g writes columns [g*D/2, (g+1)*D/2) of A1 * scale.
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
          const int col = g * (D / 2) + c * 32;
          uint32_t v[32];
          tmem_ld32(tmem + lane_off + C::TM_A1 + col, v);
          if (in_range) {
            if (valid_row) store_row32(out1 + row_off + col, v, scale);
            else store_zero32(out1 + row_off + col);
          }
        }
      } else {
        // dK (= A1 * scale) by warpgroup 0, dV (= A2) by warpgroup 1.
        const uint32_t tA = tmem + lane_off + (g == 0 ? C::TM_A1 : C::TM_A2);
        __nv_bfloat16* dst = (g == 0 ? out1 : out2) + row_off;
        const float mul = (g == 0) ? scale : 1.0f;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(tA + c * 32, v);
          if (in_range) {
            if (valid_row) store_row32(dst + c * 32, v, mul);
            else store_zero32(dst + c * 32);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar.acc_empty);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

template <int D, bool KV>
cudaError_t launch_bwd_impl(const CUtensorMap& r1, const CUtensorMap& r2, const CUtensorMap& c1,
                            const CUtensorMap& c2, void* out1, void* out2, const int* lengths, int* ws, int B,
                            int H, int L, int num_sms, cudaStream_t stream) {
  using C = BwdCfg<D, KV>;
  static bool configured[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !configured[dev]) {
    cudaError_t e =
        cudaFuncSetAttribute(bwd_kernel<D, KV>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_ALLOC);
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  const long long max_items = static_cast<long long>(B) * H * ceil_div(L, kBwdItemRows);
  const int grid = static_cast<int>(std::min<long long>(num_sms, max_items));
  bwd_kernel<D, KV><<<grid, C::THREADS, C::SMEM_ALLOC, stream>>>(
      r1, r2, c1, c2, static_cast<__nv_bfloat16*>(out1), static_cast<__nv_bfloat16*>(out2), lengths, ws, H, L);
  return cudaGetLastError();
}

cudaError_t launch_bwd_dq(int d, const CUtensorMap& tq, const CUtensorMap& tdo, const CUtensorMap& tk,
                          const CUtensorMap& tv, void* dq, const int* lengths, int* ws, int B, int H, int L,
                          int num_sms, cudaStream_t stream) {
  if (d == 64) return launch_bwd_impl<64, false>(tq, tdo, tk, tv, dq, nullptr, lengths, ws, B, H, L, num_sms, stream);
  return launch_bwd_impl<128, false>(tq, tdo, tk, tv, dq, nullptr, lengths, ws, B, H, L, num_sms, stream);
}

cudaError_t launch_bwd_dkdv(int d, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tq,
                            const CUtensorMap& tdo, void* dk, void* dv, const int* lengths, int* ws, int B, int H,
                            int L, int num_sms, cudaStream_t stream) {
  if (d == 64) return launch_bwd_impl<64, true>(tk, tv, tq, tdo, dk, dv, lengths, ws, B, H, L, num_sms, stream);
  return launch_bwd_impl<128, true>(tk, tv, tq, tdo, dk, dv, lengths, ws, B, H, L, num_sms, stream);
}

}  // namespace sigattn
