// fwd.cu -- forward sigmoid attention for sm_100a.
//
//   O = sigma(Q K^T / sqrt(d) + b) V,  b = -ln(n)   (Better Models, Faster
//   Training: Sigmoid Attention for single-cell Foundation Models, sec. 2A)
//
// Each weight is computed on its own (no row maximum, row sum or online
// rescale: sec. 2A "decoupling"), so one pass over the key blocks suffices and
// the accumulator is never rescaled.
//
// Design (one persistent CTA per SM, 608 threads):
//   warps 0-7   epilogue for query tile 0 (TMEM lanes 0..127 = its 128 rows):
//               warps 0-3 key columns 0-63, warps 4-7 key columns 64-127
//   warps 8-15  epilogue for query tile 1, split the same way
//   warp  16    TMA producer: claims work items (first blockIdx.x, then from the
//               workspace counter) and hands them to the other warps through
//               the shared-memory item ring; Q tiles once per item, then a ring
//               of K and V tiles
//   warps 17,18 one tcgen05.mma issuer per query tile (warp 17 also owns TMEM).
// A single thread issues a tcgen05.mma only every ~100 cycles, which is more
// than a 128x128x16 product takes, so each tile has its own issuing thread;
// each issuer keeps its tile's products in order (S_t(j+1) overwrites P_t(j)
// only after PV_t(j) was issued by the same thread).
// A work item is 256 query rows (two 128-row tiles) of one (b, h); both tiles
// share every K/V block that is loaded. Per key block j and tile t:
//   S_t = Q_t K_j^T          tcgen05.mma, A and B from shared memory, fp32 in TMEM
//   P_t = sigma(S_t*scale+b) epilogue warps: TMEM -> registers -> bf16 P back
//                            over the first 32 columns of each 64-column half
//   O_t += P_t V_j           tcgen05.mma with A = P_t read from TMEM
// Per tile the issue order is S_t(j), PV_t(j) (after P_t(j)), S_t(j+1), ...
// At D = 128 the two tiles' epilogues take turns (tile 1's sigmoid pass over
// block j starts when tile 0's is done, tile 0's pass over j+1 when tile 1's j
// is done): each has the MUFU pipe to itself while the tensor core works on
// the other tile, instead of both tiles running in phase (S(j+1) overwrites
// P(j) there, so a tile's next S waits for its PV). At D = 64, where P has a
// region of its own, the two tiles' warps run independently.
// TMEM: S/P of tile t at columns [128t, 128t+128), O of tile t at 256 + t*D.
// PACKED selects the input layout (padded [B][H][Lmax][d] or packed
// [total][H][d]); it changes only the TMA coordinates and output row addresses
// (RowMap), so both layouts run the same arithmetic in the same order.
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
  // At D = 64 the 512 TMEM columns leave room for P in its own region (64
  // columns of bf16 pairs per tile) instead of over S, so S(j+1) need not wait
  // for PV(j), and each tile's eight epilogue warps run independently: SEP_P.
  static constexpr bool SEP_P = (D == 64);
  static constexpr int TM_P = TM_O + 2 * D;
  static constexpr int TMEM_COLS = 512;
  static_assert(!SEP_P || TM_P + 128 <= TMEM_COLS, "TMEM budget");
  static constexpr int EPI_WARPS = 16;
  static constexpr int THREADS = (EPI_WARPS + 3) * 32;
};

template <int KST, int VST>
struct FwdBarriers {
  uint64_t q_full, q_empty;
  uint64_t k_full[KST], k_empty[KST];
  uint64_t v_full[VST], v_empty[VST];
  uint64_t s_full[2], p_full[4], o_full[2], o_empty[2];
  uint64_t epi_done[2];  // tile t's warps finished their sigmoid pass over a block
  uint64_t s_read[2];    // SEP_P: the epilogue copied tile t's S out of TMEM (S region free)
  uint64_t pv_done[2];   // SEP_P: tile t's PV products of a block completed (P region free)
  uint64_t drain[2];
  uint64_t xmax[4][2];  // softmax: the four warps of a lane quadrant wrote their row maxima (by pass parity)
  uint64_t xsum[4];     // softmax: ... their partial row sums (end of an item)
  ItemRing ring;
  uint32_t tmem_base;
  int abort;
};

// F32OUT: the output is the fp32 partial sum over the call's key range (no
// rounding to bf16), for key-range calls whose partial outputs are summed.
// SOFTMAX (D = 64, padded layout, whole sequences): softmax attention over the
// valid keys instead of the sigmoid, on the same scheduler, producer and MMA
// issuers (the counterpart that the comparison of Better Models sec. 4A
// needs): only the epilogue differs (online row maximum exchanged between the
// four warps that share a row, lazily rescaled O and row sums, O / l at the end).
template <int D, bool PACKED, bool F32OUT, bool SOFTMAX>
__global__ void __launch_bounds__((16 + 3) * 32, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, void* __restrict__ out, int* __restrict__ ws, int H, int L,
               KeyRange kr) {
  using C = FwdCfg<D>;
  static_assert(!SOFTMAX || (C::SEP_P && !PACKED && !F32OUT), "softmax: d = 64, padded layout, bf16 output");
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ FwdBarriers<C::KST, C::VST> bar;
  // Softmax only: the row maxima of a pass (two buffers, by pass parity) and
  // the row sums at the end of an item, per tile, column chunk and row.
  __shared__ float soft_max[SOFTMAX ? 2 * 4 * 128 : 1];
  __shared__ float soft_sum[SOFTMAX ? 2 * 4 * 128 : 1];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + C::OFF_Q;
  uint8_t* sK = smem + C::OFF_K;
  uint8_t* sV = smem + C::OFF_V;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  volatile int* abort_flag = &bar.abort;
  grid_dep_launch();  // the padded-row fill kernel may start beside this one

  if (threadIdx.x == 0) {
    // "empty" barriers take one arrival from each of the two issuers
    mbar_init(&bar.q_full, 1);
    mbar_init(&bar.q_empty, 2);
    for (int s = 0; s < C::KST; ++s) { mbar_init(&bar.k_full[s], 1); mbar_init(&bar.k_empty[s], 2); }
    for (int s = 0; s < C::VST; ++s) { mbar_init(&bar.v_full[s], 1); mbar_init(&bar.v_empty[s], 2); }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&bar.s_full[t], 1);
      // P of a key half: 4 warps (one per lane quadrant), or with the softmax
      // epilogue the 8 warps that cover its two 32-column chunks. S is read by
      // the tile's 8 warps, or (softmax) by all 16.
      mbar_init(&bar.p_full[2 * t], (C::SEP_P && SOFTMAX) ? 8 : 4);
      mbar_init(&bar.p_full[2 * t + 1], (C::SEP_P && SOFTMAX) ? 8 : 4);
      mbar_init(&bar.s_read[t], SOFTMAX ? C::EPI_WARPS : C::EPI_WARPS / 2);
      mbar_init(&bar.pv_done[t], 1);
      mbar_init(&bar.o_full[t], 1);
      mbar_init(&bar.o_empty[t], 8);
    }
    mbar_init(&bar.epi_done[0], 8);
    mbar_init(&bar.epi_done[1], 8);
    mbar_init(&bar.drain[0], 1);
    mbar_init(&bar.drain[1], 1);
    for (int q = 0; q < 4; ++q) {
      mbar_init(&bar.xmax[q][0], 4);
      mbar_init(&bar.xmax[q][1], 4);
      mbar_init(&bar.xsum[q], 4);
    }
    ring_init(bar.ring, 2 + C::EPI_WARPS);  // both issuers and every epilogue warp read each item
    bar.abort = 0;
    fence_mbar_init();
  }
  constexpr int kProducerWarp = C::EPI_WARPS, kMmaWarp = C::EPI_WARPS + 1;  // issuers: kMmaWarp + t
  if (warp == kMmaWarp) {
    tmem_alloc(&bar.tmem_base, C::TMEM_COLS);
    tmem_relinquish();
  }
  // The plan is written by the kernel before this one in the stream.
  grid_dep_wait();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar.tmem_base;
  const int count = ws[kHdrCount];
  const RowMap<PACKED> rm{H, L};

  if (warp == kProducerWarp) {
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
      uint32_t ist = 0, iph = 0;
      int claimed = -1;
      while (ok) {
        const Item item = next_item(ws, claimed, count);
        if (!(ok = ring_publish(bar.ring, ist, iph, item, abort_flag, ws, 100))) break;
        if (item.n < 0) break;
        const int n = item.n;
        const int hd = PACKED ? item.bh % H : 0;
        const int row0 = item.blk * (C::BM * C::NQ);
        const int ntiles = (row0 + C::BM < n) ? 2 : 1;
        const int nkb = ceil_div(range_keys(n, kr), C::BN);  // K/V rows are the range's keys
        if (!(ok = mbar_wait(&bar.q_empty, qph ^ 1, abort_flag, ws, 101))) break;
        mbar_arrive_expect_tx(&bar.q_full, ntiles * C::TILE_BYTES);
        for (int t = 0; t < ntiles; ++t)
          for (int c = 0; c < D / 64; ++c)
            tma_load_3d(sQ + t * C::TILE_BYTES + c * C::BOX_BYTES, &tm_q, &bar.q_full, c * 64,
                        rm.y(item, hd, row0 + t * C::BM), rm.z(item, row0 + t * C::BM));
        q_last = static_cast<int>(qph);
        qph ^= 1;
        for (int j = 0; j < nkb; ++j) {
          // Claim the CTA's next item two key blocks before this one ends.
          if (j == max(0, nkb - 2)) claimed = atomicAdd(ws + kHdrNext, 1);
          if (!(ok = mbar_wait(&bar.k_empty[kst], kph ^ 1, abort_flag, ws, 102))) break;
          mbar_arrive_expect_tx(&bar.k_full[kst], C::TILE_BYTES);
          for (int c = 0; c < D / 64; ++c)
            tma_load_3d(sK + kst * C::TILE_BYTES + c * C::BOX_BYTES, &tm_k, &bar.k_full[kst], c * 64,
                        rm.y(item, hd, j * C::BN), rm.z(item, j * C::BN));
          k_last[kst] = static_cast<int>(kph);
          if (++kst == C::KST) { kst = 0; kph ^= 1; }
          if (!(ok = mbar_wait(&bar.v_empty[vst], vph ^ 1, abort_flag, ws, 103))) break;
          mbar_arrive_expect_tx(&bar.v_full[vst], C::TILE_BYTES);
          for (int c = 0; c < D / 64; ++c)
            tma_load_3d(sV + vst * C::TILE_BYTES + c * C::BOX_BYTES, &tm_v, &bar.v_full[vst], c * 64,
                        rm.y(item, hd, j * C::BN), rm.z(item, j * C::BN));
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
  } else if (warp >= kMmaWarp) {
    // ------------------------------------------------------- MMA issuer of tile t
    const int t = warp - kMmaWarp;
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, C::BN, false, false);
      constexpr uint32_t idesc_o = idesc_bf16_f32(128, D, false, true);
      const uint32_t q_addr = smem_u32(sQ), k_addr = smem_u32(sK), v_addr = smem_u32(sV);
      uint32_t kst = 0, kph = 0, vst = 0, vph = 0, qph = 0;
      uint32_t pph[2] = {0, 0}, oph = 0;
      bool ok = true;
      // Descriptors are built once and advanced by adding (bytes >> 4): the
      // start-address field is the low 14 bits and smem stays below 256 KB.
      const uint64_t d_q = smem_desc_sw128(q_addr, 16, 1024) + ((t * C::TILE_BYTES) >> 4);
      const uint64_t d_k = smem_desc_sw128(k_addr, 16, 1024);
      const uint64_t d_v = smem_desc_sw128(v_addr, C::BOX_BYTES, 1024);  // MN-major view of V
      constexpr uint64_t kTile = C::TILE_BYTES >> 4;
      const uint32_t tm_s = tmem + C::TM_S + t * 128;
      const uint32_t tm_o = tmem + C::TM_O + t * D;
      // P of key half h: over the first 32 columns of S's half, or (SEP_P) in
      // its own region, 32 columns per half.
      const uint32_t tm_p = C::SEP_P ? tmem + C::TM_P + t * 64 : tm_s;
      constexpr int kPHalf = C::SEP_P ? 32 : 64;
      uint32_t srph = 0;
      bool s_pending = false;  // SEP_P: an S was issued whose copy-out has not been awaited

      auto issue_s = [&](uint32_t ks) {
        const uint64_t b0 = d_k + ks * kTile;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t off = ((kk >> 2) * C::BOX_BYTES + (kk & 3) * 32) >> 4;
          mma_ss(tm_s, d_q + off, b0 + off, idesc_s, kk > 0 ? 1u : 0u);
        }
      };
      // O_t += P_t[:, 64h : 64h+64] V_j[64h : 64h+64, :] for key half h: P of
      // that half sits in TMEM columns [128t + 64h, 128t + 64h + 32).
      auto issue_pv = [&](int h, uint32_t vs, bool acc) {
        const uint64_t b0 = d_v + vs * kTile + ((h * 64 * 128) >> 4);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_ts(tm_o, tm_p + h * kPHalf + kk * 8, b0 + ((kk * 2048) >> 4), idesc_o, (acc || kk > 0) ? 1u : 0u);
      };
      auto advance_k = [&]() { if (++kst == C::KST) { kst = 0; kph ^= 1; } };
      auto advance_v = [&]() { if (++vst == C::VST) { vst = 0; vph ^= 1; } };
      // SEP_P: before an S product overwrites the S region, the epilogue must
      // have copied out the previous S of this tile.
      auto wait_s_free = [&]() -> bool {
        if (!C::SEP_P || !s_pending) return true;
        if (!mbar_wait(&bar.s_read[t], srph, abort_flag, ws, 118)) return false;
        srph ^= 1;
        s_pending = false;
        return true;
      };

      uint32_t ist = 0, iph = 0;
      while (ok) {
        Item item;
        if (!(ok = ring_read(bar.ring, ist, iph, &item, abort_flag, ws, 110))) break;
        ring_release(bar.ring, ist, iph, true);
        if (item.n < 0) break;
        const int n = item.n;
        const int row0 = item.blk * (C::BM * C::NQ);
        const int ntiles = (row0 + C::BM < n) ? 2 : 1;
        const int nkb = ceil_div(range_keys(n, kr), C::BN);
        if (t >= ntiles) {
          // Tile 1 is fully padded in this item. Its issuer issues nothing but
          // still waits for every load and gives its arrival on every shared
          // "empty" barrier, so both issuers stay in step with the rings.
          if (!(ok = mbar_wait(&bar.q_full, qph, abort_flag, ws, 117))) break;
          qph ^= 1;
          for (int j = 0; ok && j < nkb; ++j) {
            if (!(ok = mbar_wait(&bar.k_full[kst], kph, abort_flag, ws, 117))) break;
            mma_commit(&bar.k_empty[kst]);
            advance_k();
            if (!(ok = mbar_wait(&bar.v_full[vst], vph, abort_flag, ws, 117))) break;
            mma_commit(&bar.v_empty[vst]);
            advance_v();
          }
          mma_commit(&bar.q_empty);
          continue;
        }
        if (!(ok = mbar_wait(&bar.q_full, qph, abort_flag, ws, 111))) break;
        qph ^= 1;
        if (!(ok = mbar_wait(&bar.k_full[kst], kph, abort_flag, ws, 112))) break;
        if (!(ok = wait_s_free())) break;
        tc_fence_after();
        issue_s(kst);
        s_pending = true;
        mma_commit(&bar.s_full[t]);
        if (nkb == 1) mma_commit(&bar.q_empty);
        mma_commit(&bar.k_empty[kst]);
        advance_k();

        for (int j = 0; ok && j < nkb; ++j) {
          const bool has_next = (j + 1 < nkb);
          // S(j+1) goes first when P has its own region (as soon as the
          // epilogue has copied S(j) out); otherwise it overwrites P(j) and
          // must follow PV(j).
          auto next_s = [&]() -> bool {
            if (!mbar_wait(&bar.k_full[kst], kph, abort_flag, ws, 116)) return false;
            if (!wait_s_free()) return false;
            tc_fence_after();
            issue_s(kst);
            s_pending = true;
            mma_commit(&bar.s_full[t]);
            if (j + 2 == nkb) mma_commit(&bar.q_empty);
            mma_commit(&bar.k_empty[kst]);
            advance_k();
            return true;
          };
          if (C::SEP_P && has_next && !(ok = next_s())) break;
          if (!(ok = mbar_wait(&bar.v_full[vst], vph, abort_flag, ws, 113))) break;
          for (int h = 0; h < 2; ++h) {
            if (!(ok = mbar_wait(&bar.p_full[2 * t + h], pph[h], abort_flag, ws, 114))) break;
            pph[h] ^= 1;
            if (j == 0 && h == 0) {
              if (!(ok = mbar_wait(&bar.o_empty[t], oph ^ 1, abort_flag, ws, 115))) break;
              oph ^= 1;
            }
            tc_fence_after();
            issue_pv(h, vst, j > 0 || h > 0);
          }
          if (!ok) break;
          mma_commit(&bar.v_empty[vst]);
          advance_v();
          if (C::SEP_P) mma_commit(&bar.pv_done[t]);
          if (!C::SEP_P && has_next && !(ok = next_s())) break;
        }
        if (!ok) break;
        mma_commit(&bar.o_full[t]);
      }
      // Wait for every MMA issued so far before TMEM can be released.
      int never = 0;
      mma_commit(&bar.drain[t]);
      mbar_wait(&bar.drain[t], 0, &never, ws, 119);
    }
  } else if constexpr (SOFTMAX) {
    // -------------------------------------------- softmax epilogue (D = 64)
    // Warp w covers lane quadrant qd = w & 3 and key columns [32c, 32c + 32),
    // c = w >> 2, as in the sigmoid epilogue below. Per pass (tile t, key
    // block j) each warp takes its chunk's row maximum; the four warps of a
    // quadrant exchange them through shared memory (an mbarrier per quadrant
    // and buffer parity, waited with the same bound as every other hand-off),
    // so all four hold the same block maximum and the same running maximum m.
    // m only moves when the block maximum exceeds it by more than kTau
    // (log2 units), and then O and the partial row sums l are rescaled by
    // 2^(m_old - m_new) (warps c = 0, 1 rescale the tile's 64 O columns, before
    // they signal the first P half, which the issuer waits for before the
    // block's first PV product). P = 2^(y - m) with y = s * scale * log2(e).
    // At the end of an item the four partial row sums are added through
    // shared memory and O is divided by them.
    constexpr float kTau = 8.0f;
    const int c = warp >> 2, qd = warp & 3;
    const int r = (qd << 5) + lane;
    const uint32_t lane_off = static_cast<uint32_t>(qd << 5) << 16;
    const int ot = c >> 1, oc = c & 1;
    constexpr float scale_l2e = Scale<D>::value * kLog2e;
    uint32_t sph[2] = {0, 0}, oph[2] = {0, 0}, pvph[2] = {0, 0};
    bool pv_pending[2] = {false, false};
    uint32_t pass = 0, sum_ph = 0;
    bool ok = true;
    uint32_t ist = 0, iph = 0;
    while (ok) {
      Item item;
      if (!(ok = ring_read(bar.ring, ist, iph, &item, abort_flag, ws, 120))) break;
      __syncwarp();
      ring_release(bar.ring, ist, iph, lane == 0);
      if (item.n < 0) break;
      const int n = item.n;
      const int row_base = item.blk * (C::BM * C::NQ);
      const int ntiles = (row_base + C::BM < n) ? 2 : 1;
      const int nkb = ceil_div(n, C::BN);
      float m[2] = {0.f, 0.f}, l[2] = {0.f, 0.f};
      for (int j = 0; ok && j < nkb; ++j) {
        const int valid = n - (j * C::BN + 32 * c);  // columns < valid are real keys
        for (int t = 0; t < ntiles; ++t) {
          if (!(ok = mbar_wait(&bar.s_full[t], sph[t], abort_flag, ws, 121))) break;
          sph[t] ^= 1;
          tc_fence_after();
          uint32_t a[32];
          tmem_ld32(tmem + lane_off + C::TM_S + t * 128 + 32 * c, a);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bar.s_read[t]);
          // y in log2 units; keys past n get -inf, rows past n (discarded) 0
          const bool row_ok = row_base + t * C::BM + r < n;
          float cm = -INFINITY;  // a[e] becomes y, in place
          if (valid >= 32 && row_ok) {
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const float y = __uint_as_float(a[e]) * scale_l2e;
              a[e] = __float_as_uint(y);
              cm = fmaxf(cm, y);
            }
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const float y = !row_ok ? 0.0f : (e < valid ? __uint_as_float(a[e]) * scale_l2e : -INFINITY);
              a[e] = __float_as_uint(y);
              cm = fmaxf(cm, y);
            }
          }
          float* mx = soft_max + (pass & 1) * 512;
          mx[c * 128 + r] = cm;
          __syncwarp();
          if (lane == 0) mbar_arrive(&bar.xmax[qd][pass & 1]);
          if (!(ok = mbar_wait(&bar.xmax[qd][pass & 1], (pass >> 1) & 1, abort_flag, ws, 125))) break;
          const float bm = fmaxf(fmaxf(mx[r], mx[128 + r]), fmaxf(mx[256 + r], mx[384 + r]));
          ++pass;
          // O and the P region are free once the tile's previous PV products completed.
          if (pv_pending[t]) {
            if (!(ok = mbar_wait(&bar.pv_done[t], pvph[t], abort_flag, ws, 124))) break;
            pvph[t] ^= 1;
          }
          pv_pending[t] = true;
          tc_fence_after();
          if (j == 0) {
            m[t] = bm;  // the block's first PV product overwrites O
            l[t] = 0.f;
          } else if (__any_sync(0xffffffffu, bm > m[t] + kTau)) {
            const float mn = fmaxf(m[t], bm);
            const float alpha = ex2_approx(m[t] - mn);
            m[t] = mn;
            l[t] *= alpha;
            if (c < 2) {
#pragma unroll
              for (int hf = 0; hf < 2; ++hf) {
                const uint32_t to = tmem + lane_off + C::TM_O + t * D + 32 * c + 16 * hf;
                uint32_t o[16];
                tmem_ld16(to, o);
#pragma unroll
                for (int e = 0; e < 16; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                tmem_st16(to, o);
              }
            }
          }
          uint32_t pk[16];
          float ls = 0.f;
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float p0 = ex2_approx(__uint_as_float(a[2 * e]) - m[t]);
            const float p1 = ex2_approx(__uint_as_float(a[2 * e + 1]) - m[t]);
            ls += p0 + p1;
            pk[e] = pack_bf16x2(p0, p1);
          }
          l[t] += ls;
          tmem_st16(tmem + lane_off + C::TM_P + t * 64 + 16 * c, pk);
          tmem_st_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bar.p_full[2 * t + (c >> 1)]);
        }
      }
      if (!ok) break;
      // Row sums: the four partials of each row, added through shared memory.
      for (int t = 0; t < ntiles; ++t) soft_sum[t * 512 + c * 128 + r] = l[t];
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar.xsum[qd]);
      if (!(ok = mbar_wait(&bar.xsum[qd], sum_ph, abort_flag, ws, 126))) break;
      sum_ph ^= 1;
      const int row = row_base + ot * C::BM + r;
      const size_t orow = rm.offset(item, 0, row, D) + 32 * oc;
      if (ot >= ntiles) {  // tile fully padded: its rows of O are zero
        if (rm.writes(row, n)) store_zero_out32<false>(out, orow);
        continue;
      }
      const float* ps = soft_sum + ot * 512;
      const float inv_l = 1.0f / (ps[r] + ps[128 + r] + ps[256 + r] + ps[384 + r]);
      if (!(ok = mbar_wait(&bar.o_full[ot], oph[ot], abort_flag, ws, 122))) break;
      oph[ot] ^= 1;
      tc_fence_after();
      uint32_t v[32];
      tmem_ld32(tmem + lane_off + C::TM_O + ot * D + 32 * oc, v);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar.o_empty[ot]);
      if (rm.writes(row, n)) store_out32<false>(out, orow, v, inv_l, row >= n);
    }
  } else if constexpr (C::SEP_P) {
    // ------------------------------------------------- epilogue (D = 64, SEP_P)
    // Two independent groups of eight warps, one per query tile (warps 0-7
    // tile 0, 8-15 tile 1): since P has its own region, a tile's S(j+1) is
    // issued as soon as its warps have copied S(j) out, so the tiles need not
    // take turns, and the four warps that share a scheduler (two per tile)
    // work at independent points of their passes, which keeps the MUFU queue
    // fed. Warp w reads TMEM lane quadrant w & 3 and the 64-column half
    // h = (w >> 2) & 1 of each key block, as two 32-column chunks; the P of
    // chunk cc (bf16 pairs) goes to columns [16cc, 16cc + 16) of the tile's P
    // region. At the end of an item warp w reads out its tile's output columns
    // [32h, 32h + 32). (Sixteen warps per pass with the tiles taking turns,
    // 32 columns per warp, measured 3.7 % slower on the unpadded sweep.)
    const int c = warp >> 2;
    const int r = ((warp & 3) << 5) + lane;        // row within a tile = TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) << 5) << 16;
    const int ot = c >> 1, oc = c & 1;
    constexpr float scale_l2e = Scale<D>::value * kLog2e;
    uint32_t sph[2] = {0, 0}, oph[2] = {0, 0}, pvph[2] = {0, 0};
    bool pv_pending[2] = {false, false};  // a P of the tile was written whose PV has not been awaited
    bool ok = true;
    uint32_t ist = 0, iph = 0;
    while (ok) {
      Item item;
      if (!(ok = ring_read(bar.ring, ist, iph, &item, abort_flag, ws, 120))) break;
      __syncwarp();
      ring_release(bar.ring, ist, iph, lane == 0);
      if (item.n < 0) break;
      const int n = item.n;
      const int row_base = item.blk * (C::BM * C::NQ);
      const int ntiles = (row_base + C::BM < n) ? 2 : 1;
      const int nk = range_keys(n, kr);
      const int nkb = ceil_div(nk, C::BN);
      const float neg_log2n = -__log2f(static_cast<float>(n));  // bias * log2(e)
      const int t = ot;  // this warp's tile; the two tiles' warps run independently
      const int h = oc;  // its 64-column half of each key block (two 32-column chunks)
      // A padded row's weights only reach its own output row, which is
      // discarded: such rows are not masked, and they take no part in the
      // warp's choice of sigmoid form (so their values never change a valid
      // output's bits).
      const bool row_ok = row_base + t * C::BM + r < n;
      // One pass over key block j. MASKED (the last block, the only one that
      // can hold keys past the sequence): those scores are set to -inf before
      // the sigmoid; the other passes carry no masking code at all.
      auto pass = [&](const int j, auto masked) -> bool {
        constexpr bool MASKED = decltype(masked)::value;
        if (!mbar_wait(&bar.s_full[t], sph[t], abort_flag, ws, 121)) return false;
        sph[t] ^= 1;
        for (int i = 0; i < 2; ++i) {
          const int cc = 2 * h + i;
          tc_fence_after();
          uint32_t a[32];
          tmem_ld32(tmem + lane_off + C::TM_S + t * 128 + 32 * cc, a);
          if (i == 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar.s_read[t]);
          }
          uint32_t pk[16];
          if constexpr (MASKED) mask_scores(a, nk - (j * C::BN + 32 * cc), true);  // columns < that are keys
          sigmoid32<false>(a, scale_l2e, neg_log2n, nullptr, row_ok);
#pragma unroll
          for (int e = 0; e < 16; ++e) pk[e] = pack_bf16x2(__uint_as_float(a[2 * e]), __uint_as_float(a[2 * e + 1]));
          // The P region is free once the tile's previous PV products completed.
          if (i == 0 && pv_pending[t]) {
            if (!mbar_wait(&bar.pv_done[t], pvph[t], abort_flag, ws, 124)) return false;
            pvph[t] ^= 1;
          }
          pv_pending[t] = true;
          tc_fence_after();
          tmem_st16(tmem + lane_off + C::TM_P + t * 64 + 16 * cc, pk);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar.p_full[2 * t + h]);
        return true;
      };
      if (t < ntiles) {
        for (int j = 0; ok && j + 1 < nkb; ++j) ok = pass(j, std::false_type{});
        if (ok) ok = pass(nkb - 1, std::true_type{});
      }
      if (!ok) break;
      const int row = row_base + ot * C::BM + r;
      const size_t orow = rm.offset(item, PACKED ? item.bh % H : 0, row, D) + 32 * oc;
      if (ot >= ntiles) {  // tile fully padded: its rows of O are zero (padded layout)
        if (rm.writes(row, n)) store_zero_out32<F32OUT>(out, orow);
        continue;
      }
      if (!(ok = mbar_wait(&bar.o_full[ot], oph[ot], abort_flag, ws, 122))) break;
      oph[ot] ^= 1;
      tc_fence_after();
      uint32_t v[32];
      tmem_ld32(tmem + lane_off + C::TM_O + ot * D + 32 * oc, v);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar.o_empty[ot]);
      if (rm.writes(row, n)) store_out32<F32OUT>(out, orow, v, 1.0f, row >= n);
    }
  } else {
    // ------------------------------------------------------------- epilogue
    const int t = warp >> 3;                       // query tile of this warp
    const int h = (warp >> 2) & 1;                 // key half (64 columns) of this warp
    const int r = ((warp & 3) << 5) + lane;        // row within the tile = TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) << 5) << 16;
    const uint32_t tS = tmem + lane_off + C::TM_S + t * 128 + h * 64;
    const uint32_t tO = tmem + lane_off + C::TM_O + t * D + h * (D / 2);
    constexpr float scale_l2e = Scale<D>::value * kLog2e;
    uint32_t sph = 0, oph = 0, turn_ph = 0;
    bool ok = true;
    uint32_t ist = 0, iph = 0;
    while (ok) {
      Item item;
      if (!(ok = ring_read(bar.ring, ist, iph, &item, abort_flag, ws, 120))) break;
      __syncwarp();
      ring_release(bar.ring, ist, iph, lane == 0);
      if (item.n < 0) break;
      const int n = item.n;
      const bool two_tiles = item.blk * (C::BM * C::NQ) + C::BM < n;
      const int row0 = item.blk * (C::BM * C::NQ) + t * C::BM;
      const int row = row0 + r;
      const size_t orow = rm.offset(item, PACKED ? item.bh % H : 0, row, D) + h * (D / 2);
      if (row0 >= n) {  // tile fully padded: its rows of O are zero (padded layout)
        if (rm.writes(row, n)) {
#pragma unroll
          for (int c = 0; c < D / 64; ++c) store_zero_out32<F32OUT>(out, orow + c * 32);
        }
        continue;
      }
      const int nk = range_keys(n, kr);
      const int nkb = ceil_div(nk, C::BN);
      const float neg_log2n = -__log2f(static_cast<float>(n));  // bias * log2(e)
      // Padded rows are not masked: their weights reach only their own,
      // discarded output rows, and they take no part in the choice of
      // sigmoid form. Only the last block can hold keys past the sequence:
      // it alone runs the MASKED pass, whose scores of those keys are set to
      // -inf before the sigmoid.
      const bool row_ok = row < n;
      auto pass = [&](const int j, auto masked) -> bool {
        constexpr bool MASKED = decltype(masked)::value;
        if (!mbar_wait(&bar.s_full[t], sph, abort_flag, ws, 121)) return false;
        sph ^= 1;
        // Take turns with the other tile (two-tile items only): tile 1 waits
        // for tile 0's pass over block j, tile 0 for tile 1's pass over j-1.
        if (two_tiles && (t == 1 || j > 0)) {
          if (!mbar_wait(&bar.epi_done[1 - t], turn_ph, abort_flag, ws, 123)) return false;
          turn_ph ^= 1;
        }
        tc_fence_after();
        // The half's 64 keys in two 32-column chunks; P of chunk c goes to
        // TMEM columns [16c, 16c + 16) of the half, which hold S values this
        // thread has already read (chunk 0's).
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t a[32];
          tmem_ld32(tS + 32 * c, a);
          uint32_t pk[16];
          if constexpr (MASKED) mask_scores(a, nk - (j * C::BN + h * 64 + 32 * c), true);  // columns < that are keys
          sigmoid32<false>(a, scale_l2e, neg_log2n, nullptr, row_ok);
#pragma unroll
          for (int e = 0; e < 16; ++e) pk[e] = pack_bf16x2(__uint_as_float(a[2 * e]), __uint_as_float(a[2 * e + 1]));
          tmem_st16(tS + 16 * c, pk);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&bar.p_full[2 * t + h]);
          // Hand the turn over: every pass of tile 0 is awaited by tile 1;
          // tile 1's last pass of the item has no successor to wait for it.
          if (two_tiles && (t == 0 || j + 1 < nkb)) mbar_arrive(&bar.epi_done[t]);
        }
        return true;
      };
      for (int j = 0; ok && j + 1 < nkb; ++j) ok = pass(j, std::false_type{});
      if (ok) ok = pass(nkb - 1, std::true_type{});
      if (!ok) break;
      if (!(ok = mbar_wait(&bar.o_full[t], oph, abort_flag, ws, 122))) break;
      oph ^= 1;
      tc_fence_after();
      // This warp's D/2 columns of O: copy them all out, release O, then store.
      uint32_t v[D / 64][32];
#pragma unroll
      for (int c = 0; c < D / 64; ++c) tmem_ld32_async(tO + c * 32, v[c]);
#pragma unroll
      for (int c = 0; c < D / 64; ++c) tmem_ld_wait32(v[c]);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar.o_empty[t]);
      if (rm.writes(row, n)) {
#pragma unroll
        for (int c = 0; c < D / 64; ++c) store_out32<F32OUT>(out, orow + c * 32, v[c], 1.0f, row >= n);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

template <int D, bool PACKED, bool F32OUT, bool SOFTMAX = false>
cudaError_t launch_fwd_impl(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, void* o, int* ws,
                            int B, int H, int L, KeyRange kr, int num_sms, cudaStream_t stream) {
  using C = FwdCfg<D>;
  static PerDeviceOnce attr;
  const cudaError_t e = attr.run([] {
    return cudaFuncSetAttribute(fwd_kernel<D, PACKED, F32OUT, SOFTMAX>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                C::SMEM_ALLOC);
  });
  if (e != cudaSuccess) return e;
  const long long max_items = static_cast<long long>(B) * H * ceil_div(L, kFwdItemRows);
  const int grid = static_cast<int>(std::min<long long>(num_sms, max_items));
  return launch_programmatic(fwd_kernel<D, PACKED, F32OUT, SOFTMAX>, dim3(grid), dim3(C::THREADS), C::SMEM_ALLOC,
                             stream, tq, tk, tv, o, ws, H, L, kr);
}

// The softmax counterpart (d = 64, padded layout).
cudaError_t launch_softmax_fwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, void* o, int* ws,
                               int B, int H, int L, int num_sms, cudaStream_t stream) {
  return launch_fwd_impl<64, false, false, true>(tq, tk, tv, o, ws, B, H, L, KeyRange{0, L}, num_sms, stream);
}

// L is Lmax for the padded layout and the longest sequence for the packed one.
// kr: the keys covered (whole sequences: {0, L}); f32out: write the fp32
// partial sum over those keys (padded layout only).
cudaError_t launch_fwd(int d, bool packed, bool f32out, const CUtensorMap& tq, const CUtensorMap& tk,
                       const CUtensorMap& tv, void* o, int* ws, int B, int H, int L, KeyRange kr, int num_sms,
                       cudaStream_t stream) {
  if (packed) {
    if (d == 64) return launch_fwd_impl<64, true, false>(tq, tk, tv, o, ws, B, H, L, kr, num_sms, stream);
    return launch_fwd_impl<128, true, false>(tq, tk, tv, o, ws, B, H, L, kr, num_sms, stream);
  }
  if (f32out) {
    if (d == 64) return launch_fwd_impl<64, false, true>(tq, tk, tv, o, ws, B, H, L, kr, num_sms, stream);
    return launch_fwd_impl<128, false, true>(tq, tk, tv, o, ws, B, H, L, kr, num_sms, stream);
  }
  if (d == 64) return launch_fwd_impl<64, false, false>(tq, tk, tv, o, ws, B, H, L, kr, num_sms, stream);
  return launch_fwd_impl<128, false, false>(tq, tk, tv, o, ws, B, H, L, kr, num_sms, stream);
}

}  // namespace sigattn
