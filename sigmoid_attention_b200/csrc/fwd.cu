// fwd.cu -- forward sigmoid attention for sm_100a.
//
//   O = sigma(Q K^T / sqrt(d) + b) V,  b = -ln(n)   (Better Models, Faster
//   Training: Sigmoid Attention for single-cell Foundation Models, sec. 2A)
//
// Each weight is computed on its own (no row maximum, row sum or online
// rescale: sec. 2A "decoupling"), so one pass over the key blocks suffices and
// the accumulator is never rescaled.
//
// Design (one persistent CTA per SM, 320 threads):
//   warps 0-3  epilogue for query tile 0 (TMEM lanes 0..127 = its 128 rows)
//   warps 4-7  epilogue for query tile 1
//   warp  8    TMA producer: Q tiles once per item, then a ring of K and V tiles
//   warp  9    TMEM allocator and the single thread that issues tcgen05.mma
// A work item is 256 query rows (two 128-row tiles) of one (b, h); both tiles
// share every K/V block that is loaded. Per key block j and tile t:
//   S_t = Q_t K_j^T          tcgen05.mma, A and B from shared memory, fp32 in TMEM
//   P_t = sigma(S_t*scale+b) epilogue warps: TMEM -> registers -> bf16 P back
//                            into the first 64 columns of S_t's TMEM region
//   O_t += P_t V_j           tcgen05.mma with A = P_t read from TMEM
// The MMA issue order S0(j), S1(j), PV0(j), S0(j+1), PV1(j), S1(j+1), ... lets
// one tile's epilogue run while the tensor core works on the other tile.
// TMEM: S/P of tile t at columns [128t, 128t+128), O of tile t at 256 + t*D.
#include "common.cuh"

namespace sigattn {

template <int D>
struct FwdCfg {
  static constexpr int BM = 128;
  static constexpr int NQ = 2;
  static constexpr int BN = kColBlock;
  static constexpr int KST = (D == 128) ? 2 : 3;
  static constexpr int VST = (D == 128) ? 2 : 3;
  static constexpr int BOX_BYTES = 128 * 64 * 2;           // one [128 rows][64 cols] TMA box
  static constexpr int TILE_BYTES = 128 * D * 2;           // [128][D] = D/64 boxes
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + NQ * TILE_BYTES;
  static constexpr int OFF_V = OFF_K + KST * TILE_BYTES;
  static constexpr int SMEM_BYTES = OFF_V + VST * TILE_BYTES;
  static constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;     // slack for 1024-byte alignment
  static constexpr int TM_S = 0;
  static constexpr int TM_O = 256;
  static constexpr int TMEM_COLS = 512;
  static constexpr int THREADS = 320;
};

template <int KST, int VST>
struct FwdBarriers {
  uint64_t q_full, q_empty;
  uint64_t k_full[KST], k_empty[KST];
  uint64_t v_full[VST], v_empty[VST];
  uint64_t s_full[2], p_full[2], o_full[2], o_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

template <int D>
__global__ void __launch_bounds__(320, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, __nv_bfloat16* __restrict__ out,
               const int* __restrict__ lengths, int* __restrict__ ws, int H, int L) {
  using C = FwdCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ FwdBarriers<C::KST, C::VST> bar;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + C::OFF_Q;
  uint8_t* sK = smem + C::OFF_K;
  uint8_t* sV = smem + C::OFF_V;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  volatile int* abort_flag = &bar.abort;

  if (threadIdx.x == 0) {
    mbar_init(&bar.q_full, 1);
    mbar_init(&bar.q_empty, 1);
    for (int s = 0; s < C::KST; ++s) { mbar_init(&bar.k_full[s], 1); mbar_init(&bar.k_empty[s], 1); }
    for (int s = 0; s < C::VST; ++s) { mbar_init(&bar.v_full[s], 1); mbar_init(&bar.v_empty[s], 1); }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&bar.s_full[t], 1);
      mbar_init(&bar.p_full[t], 4);
      mbar_init(&bar.o_full[t], 1);
      mbar_init(&bar.o_empty[t], 4);
    }
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
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      uint32_t kst = 0, kph = 0, vst = 0, vph = 0, qph = 0;
      // Parity of the last load issued into each slot (-1: none), so that an
      // aborting producer can wait for its own copies in flight.
      int k_last[C::KST], v_last[C::VST], q_last = -1;
      for (int s = 0; s < C::KST; ++s) k_last[s] = -1;
      for (int s = 0; s < C::VST; ++s) v_last[s] = -1;
      bool ok = true;
      for (int it = blockIdx.x; ok && it < count; it += gridDim.x) {
        const Item item = load_item(ws, it);
        const int n = load_len(lengths, item.bh / H, L);
        const int row0 = item.blk * (C::BM * C::NQ);
        const int ntiles = (row0 + C::BM < n) ? 2 : 1;
        const int nkb = ceil_div(n, C::BN);
        if (!(ok = mbar_wait(&bar.q_empty, qph ^ 1, abort_flag, ws, 101))) break;
        mbar_arrive_expect_tx(&bar.q_full, ntiles * C::TILE_BYTES);
        for (int t = 0; t < ntiles; ++t)
          for (int c = 0; c < D / 64; ++c)
            tma_load_3d(sQ + t * C::TILE_BYTES + c * C::BOX_BYTES, &tm_q, &bar.q_full, c * 64, row0 + t * C::BM,
                        item.bh);
        q_last = static_cast<int>(qph);
        qph ^= 1;
        for (int j = 0; j < nkb; ++j) {
          if (!(ok = mbar_wait(&bar.k_empty[kst], kph ^ 1, abort_flag, ws, 102))) break;
          mbar_arrive_expect_tx(&bar.k_full[kst], C::TILE_BYTES);
          for (int c = 0; c < D / 64; ++c)
            tma_load_3d(sK + kst * C::TILE_BYTES + c * C::BOX_BYTES, &tm_k, &bar.k_full[kst], c * 64, j * C::BN,
                        item.bh);
          k_last[kst] = static_cast<int>(kph);
          if (++kst == C::KST) { kst = 0; kph ^= 1; }
          if (!(ok = mbar_wait(&bar.v_empty[vst], vph ^ 1, abort_flag, ws, 103))) break;
          mbar_arrive_expect_tx(&bar.v_full[vst], C::TILE_BYTES);
          for (int c = 0; c < D / 64; ++c)
            tma_load_3d(sV + vst * C::TILE_BYTES + c * C::BOX_BYTES, &tm_v, &bar.v_full[vst], c * 64, j * C::BN,
                        item.bh);
          v_last[vst] = static_cast<int>(vph);
          if (++vst == C::VST) { vst = 0; vph ^= 1; }
        }
      }
      if (!ok) {  // aborting: let the copies in flight land before the CTA exits
        int never = 0;
        volatile int* no_abort = &never;
        for (int s = 0; s < C::KST; ++s)
          if (k_last[s] >= 0) mbar_wait(&bar.k_full[s], k_last[s], no_abort, nullptr, 0);
        for (int s = 0; s < C::VST; ++s)
          if (v_last[s] >= 0) mbar_wait(&bar.v_full[s], v_last[s], no_abort, nullptr, 0);
        if (q_last >= 0) mbar_wait(&bar.q_full, q_last, no_abort, nullptr, 0);
      }
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, C::BN, false, false);
      constexpr uint32_t idesc_o = idesc_bf16_f32(128, D, false, true);
      const uint32_t q_addr = smem_u32(sQ), k_addr = smem_u32(sK), v_addr = smem_u32(sV);
      uint32_t kst = 0, kph = 0, vst = 0, vph = 0, qph = 0;
      uint32_t pph[2] = {0, 0}, oph[2] = {0, 0};
      bool ok = true;

      auto issue_s = [&](int t, uint32_t ks) {
        const uint32_t d_tmem = tmem + C::TM_S + t * 128;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::BOX_BYTES + (kk & 3) * 32;
          const uint64_t a = smem_desc_sw128(q_addr + t * C::TILE_BYTES + off, 16, 1024);
          const uint64_t b = smem_desc_sw128(k_addr + ks * C::TILE_BYTES + off, 16, 1024);
          mma_ss(d_tmem, a, b, idesc_s, kk > 0 ? 1u : 0u);
        }
      };
      auto issue_pv = [&](int t, uint32_t vs, bool acc) {
        const uint32_t d_tmem = tmem + C::TM_O + t * D;
        const uint32_t a_tmem = tmem + C::TM_S + t * 128;
#pragma unroll
        for (int kk = 0; kk < C::BN / 16; ++kk) {
          const uint64_t b = smem_desc_sw128(v_addr + vs * C::TILE_BYTES + kk * 2048, C::BOX_BYTES, 1024);
          mma_ts(d_tmem, a_tmem + kk * 8, b, idesc_o, (acc || kk > 0) ? 1u : 0u);
        }
      };

      for (int it = blockIdx.x; ok && it < count; it += gridDim.x) {
        const Item item = load_item(ws, it);
        const int n = load_len(lengths, item.bh / H, L);
        const int row0 = item.blk * (C::BM * C::NQ);
        const int ntiles = (row0 + C::BM < n) ? 2 : 1;
        const int nkb = ceil_div(n, C::BN);
        if (!(ok = mbar_wait(&bar.q_full, qph, abort_flag, ws, 111))) break;
        qph ^= 1;
        if (!(ok = mbar_wait(&bar.k_full[kst], kph, abort_flag, ws, 112))) break;
        tc_fence_after();
        for (int t = 0; t < ntiles; ++t) {
          issue_s(t, kst);
          mma_commit(&bar.s_full[t]);
        }
        if (nkb == 1) mma_commit(&bar.q_empty);
        mma_commit(&bar.k_empty[kst]);
        if (++kst == C::KST) { kst = 0; kph ^= 1; }

        for (int j = 0; ok && j < nkb; ++j) {
          const bool has_next = (j + 1 < nkb);
          if (!(ok = mbar_wait(&bar.v_full[vst], vph, abort_flag, ws, 113))) break;
          tc_fence_after();
          for (int t = 0; t < ntiles; ++t) {
            if (!(ok = mbar_wait(&bar.p_full[t], pph[t], abort_flag, ws, 114))) break;
            pph[t] ^= 1;
            if (j == 0) {
              if (!(ok = mbar_wait(&bar.o_empty[t], oph[t] ^ 1, abort_flag, ws, 115))) break;
              oph[t] ^= 1;
            }
            tc_fence_after();
            issue_pv(t, vst, j > 0);
            if (has_next) {
              if (t == 0) {
                if (!(ok = mbar_wait(&bar.k_full[kst], kph, abort_flag, ws, 116))) break;
                tc_fence_after();
              }
              issue_s(t, kst);
              mma_commit(&bar.s_full[t]);
            }
          }
          if (!ok) break;
          if (has_next) {
            if (j + 2 == nkb) mma_commit(&bar.q_empty);
            mma_commit(&bar.k_empty[kst]);
            if (++kst == C::KST) { kst = 0; kph ^= 1; }
          }
          mma_commit(&bar.v_empty[vst]);
          if (++vst == C::VST) { vst = 0; vph ^= 1; }
        }
        if (!ok) break;
        for (int t = 0; t < ntiles; ++t) mma_commit(&bar.o_full[t]);
      }
      // Wait for every MMA issued so far before TMEM can be released.
      int never = 0;
      mma_commit(&bar.drain);
      mbar_wait(&bar.drain, 0, &never, ws, 119);
    }
  } else {
    // ------------------------------------------------------------- epilogue
    const int t = warp >> 2;                       // query tile of this warpgroup
    const int r = ((warp & 3) << 5) + lane;        // row within the tile = TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) << 5) << 16;
    const uint32_t tS = tmem + lane_off + C::TM_S + t * 128;
    const uint32_t tO = tmem + lane_off + C::TM_O + t * D;
    constexpr float half_scale = 0.5f * Scale<D>::value;
    uint32_t sph = 0, oph = 0;
    bool ok = true;
    for (int it = blockIdx.x; ok && it < count; it += gridDim.x) {
      const Item item = load_item(ws, it);
      const int n = load_len(lengths, item.bh / H, L);
      const int row0 = item.blk * (C::BM * C::NQ) + t * C::BM;
      const int row = row0 + r;
      __nv_bfloat16* orow = out + (static_cast<size_t>(item.bh) * L + row) * D;
      if (row0 >= n) {  // tile fully padded: its rows of O are zero
        if (row < L) store_zero_row<D>(orow);
        continue;
      }
      const int nkb = ceil_div(n, C::BN);
      const float half_bias = -0.5f * __logf(static_cast<float>(n));
      for (int j = 0; j < nkb; ++j) {
        if (!(ok = mbar_wait(&bar.s_full[t], sph, abort_flag, ws, 121))) break;
        sph ^= 1;
        tc_fence_after();
        const int valid = n - j * C::BN;  // columns < valid are real keys
#pragma unroll
        for (int c = 0; c < 4; c += 2) {
          uint32_t a[32], b[32];
          tmem_ld32x2(tS + c * 32, tS + (c + 1) * 32, a, b);
          uint32_t pa[16], pb[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            float p0 = sigmoid_from_score(__uint_as_float(a[2 * e]), half_scale, half_bias);
            float p1 = sigmoid_from_score(__uint_as_float(a[2 * e + 1]), half_scale, half_bias);
            float p2 = sigmoid_from_score(__uint_as_float(b[2 * e]), half_scale, half_bias);
            float p3 = sigmoid_from_score(__uint_as_float(b[2 * e + 1]), half_scale, half_bias);
            if (valid < C::BN) {
              const int col = c * 32 + 2 * e;
              p0 = (col < valid) ? p0 : 0.f;
              p1 = (col + 1 < valid) ? p1 : 0.f;
              p2 = (col + 32 < valid) ? p2 : 0.f;
              p3 = (col + 33 < valid) ? p3 : 0.f;
            }
            pa[e] = pack_bf16x2(p0, p1);
            pb[e] = pack_bf16x2(p2, p3);
          }
          // P for columns [32c, 32c+64) goes to TMEM columns [16c, 16c+32),
          // which only overlap S columns this thread has already read.
          tmem_st16(tS + c * 16, pa);
          tmem_st16(tS + c * 16 + 16, pb);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar.p_full[t]);
      }
      if (!ok) break;
      if (!(ok = mbar_wait(&bar.o_full[t], oph, abort_flag, ws, 122))) break;
      oph ^= 1;
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(tO + c * 32, v);
        if (row < L) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
          if (row < n) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              dst[q] = make_uint4(pack_bf16x2(__uint_as_float(v[8 * q + 0]), __uint_as_float(v[8 * q + 1])),
                                  pack_bf16x2(__uint_as_float(v[8 * q + 2]), __uint_as_float(v[8 * q + 3])),
                                  pack_bf16x2(__uint_as_float(v[8 * q + 4]), __uint_as_float(v[8 * q + 5])),
                                  pack_bf16x2(__uint_as_float(v[8 * q + 6]), __uint_as_float(v[8 * q + 7])));
            }
          } else {
#pragma unroll
            for (int q = 0; q < 4; ++q) dst[q] = make_uint4(0, 0, 0, 0);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar.o_empty[t]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

template <int D>
cudaError_t launch_fwd_impl(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, void* o,
                            const int* lengths, int* ws, int B, int H, int L, int num_sms, cudaStream_t stream) {
  using C = FwdCfg<D>;
  static bool configured[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(fwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_ALLOC);
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  const long long max_items = static_cast<long long>(B) * H * ceil_div(L, kFwdItemRows);
  const int grid = static_cast<int>(std::min<long long>(num_sms, max_items));
  fwd_kernel<D><<<grid, C::THREADS, C::SMEM_ALLOC, stream>>>(tq, tk, tv, static_cast<__nv_bfloat16*>(o), lengths,
                                                             ws, H, L);
  return cudaGetLastError();
}

cudaError_t launch_fwd(int d, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, void* o,
                       const int* lengths, int* ws, int B, int H, int L, int num_sms, cudaStream_t stream) {
  if (d == 64) return launch_fwd_impl<64>(tq, tk, tv, o, lengths, ws, B, H, L, num_sms, stream);
  return launch_fwd_impl<128>(tq, tk, tv, o, lengths, ws, B, H, L, num_sms, stream);
}

}  // namespace sigattn
