// common.cuh -- constants and small device helpers shared by the plan, forward
// and backward kernels of the sigmoid-attention library.
#pragma once

#include <algorithm>
#include <cstdint>
#include <mutex>
#include <type_traits>
#include <utility>
#include <cuda_bf16.h>

#include "sm100.cuh"

namespace sigattn {

// Rows of one work item, per call kind. A work item is one block of
// consecutive rows of one (batch, head) slice holding >= 1 valid token:
//  * forward: 256 query rows (two 128-row query tiles sharing each K/V block),
//  * dQ:      128 query rows,
//  * dK/dV:   128 key rows.
// Every inner loop walks blocks of columns (keys for forward/dQ, queries for
// dK/dV; 128 wide, 64 for dK/dV at d = 128) only up to the last block holding
// a valid token, so fully padded blocks are never touched on either side.
enum Kind : int { kKindFwd = 0, kKindDq = 1, kKindDkdv = 2 };
constexpr int kFwdItemRows = 256;
constexpr int kBwdItemRows = 128;
constexpr int kColBlock = 128;
constexpr int kMaxBatch = 4096;        // sequences per call (plan runs in one CTA)
constexpr int kMaxLen = 1 << 20;       // Lmax bound (TMA coordinates are int32)

__host__ __device__ constexpr int item_rows(int kind) { return kind == kKindFwd ? kFwdItemRows : kBwdItemRows; }

// Columns per block streamed by a backward kernel: 128, except 64 for dK/dV
// with d = 128 (its TMEM budget).
__host__ __device__ constexpr int bwd_col_block(bool kv, int d) { return (kv && d == 128) ? 64 : 128; }

__host__ __device__ inline int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Valid length of sequence b, or 0 if the caller's value is outside [0, L]
// (the plan flags that case in the workspace header).
__device__ __forceinline__ int load_len(const int* lengths, int b, int L) {
  const int n = __ldg(lengths + b);
  return (n < 0 || n > L) ? 0 : n;
}

// The keys a call covers: positions [begin, begin + count) of every
// sequence. The ordinary calls cover whole sequences ({0, Lmax}); a call over
// a key range computes the contribution of those keys only (the partial sums
// of a key-sharded forward and dQ; the dK/dV rows of those keys). The bias
// -ln n_b always uses the sequence's full length n_b.
struct KeyRange {
  int begin, count;
};

// How a backward kernel is tied to the kernels around it: `err` receives the
// error words (nullptr: the header of the kernel's own plan), and `overlap`
// runs the dK/dV kernel of a whole-backward call beside the dQ kernel
// launched before it (see bwd.cu).
struct BwdLink {
  int* err = nullptr;
  bool overlap = false;
};

// One work list that the plan kernel builds: its kind, key range and
// workspace region (header and list).
struct PlanRegion {
  int kind;
  KeyRange kr;
  int* ws;
};

// Valid keys of a sequence of n tokens inside the range.
__host__ __device__ inline int range_keys(int n, KeyRange kr) {
  return n - kr.begin < 0 ? 0 : (n - kr.begin > kr.count ? kr.count : n - kr.begin);
}

// Rows that get work items: forward/dQ all n query rows when the range holds
// a valid key (none otherwise); dK/dV the range's valid keys.
__host__ __device__ inline int work_rows(int kind, int n, KeyRange kr) {
  const int nk = range_keys(n, kr);
  return kind == kKindDkdv ? nk : (nk > 0 ? n : 0);
}

// Columns each item walks: forward/dQ the range's valid keys; dK/dV all n
// queries. (For whole-sequence calls both are n.)
__host__ __device__ inline int work_cols(int kind, int n, KeyRange kr) {
  return kind == kKindDkdv ? n : range_keys(n, kr);
}

// Where a call's zero fill writes: rows [cover, out_rows) of every (b, h)
// slice of an output with `chunks_per_row` 16-byte chunks per row, cover being
// the rows its work items write (work_rows rounded up to whole items).
struct FillGeom {
  int H, L;            // heads; the bound on valid lengths (Lmax)
  int out_rows;        // rows per slice of the output (Lmax, or the key range's count for dK/dV)
  int chunks_per_row;  // d * element bytes / 16
  int kind, item_rows;
  KeyRange kr;
  __device__ __forceinline__ int cover(int n) const {
    return min(out_rows, ceil_div(work_rows(kind, n, kr), item_rows) * item_rows);
  }
};

// One work item as the plan stores it: 16 bytes {b * H + h, row block, n_b,
// start_b}, so a kernel learns the item, its sequence's valid length and (for
// packed inputs) the sequence's first token from one load.
struct Item {
  int bh;     // b * H + h
  int blk;    // row-block index within the slice
  int n;      // valid length of sequence b
  int start;  // packed layout: index of the sequence's first token (0 when padded)
};

__device__ __forceinline__ Item load_item(const int* ws, int idx) {
  const int4 v = reinterpret_cast<const int4*>(ws + kHeaderWords)[idx];
  return Item{v.x, v.y, v.z, v.w};
}

// Where the rows of a (b, h) slice live, for both input layouts.
//  padded [B][H][Lmax][d]: TMA view {d, Lmax, B*H}; row r of slice bh is at
//    (y, z) = (r, bh). Rows n_b <= r < Lmax are padding and are written as zeros.
//  packed [total][H][d] (sequence b holds tokens start_b .. start_b + n_b - 1):
//    TMA view {d, H, total}; row r is at (y, z) = (h, start_b + r). Rows r >= n_b
//    belong to the next sequence and are never written.
template <bool PACKED>
struct RowMap {
  int H, L;
  __device__ __forceinline__ int y(const Item& it, int h, int row) const { return PACKED ? h : row; }
  __device__ __forceinline__ int z(const Item& it, int row) const { return PACKED ? it.start + row : it.bh; }
  // Element offset of the row in an output tensor of head size D.
  __device__ __forceinline__ size_t offset(const Item& it, int h, int row, int D) const {
    return PACKED ? (static_cast<size_t>(it.start + row) * H + h) * D : (static_cast<size_t>(it.bh) * L + row) * D;
  }
  // Whether the item's epilogue writes this row (zeros when row >= n).
  __device__ __forceinline__ bool writes(int row, int n) const { return PACKED ? row < n : row < L; }
};

constexpr Item kNoItem{0, 0, -1, 0};  // end of the work list

// Dynamic longest-processing-time-first scheduling. The plan lists the items
// longest first; each CTA's producer takes item blockIdx.x first and every
// later one from the claim counter in the workspace header, so a CTA gets the
// next item of the list when it is ready for one. The producer hands each
// item to the CTA's other roles through this two-slot ring in shared memory
// (so they never wait on a global load for it); after the last item it
// publishes kNoItem.
struct ItemRing {
  int4 slot[2];
  uint64_t full[2];   // count 1: the producer wrote the slot
  uint64_t empty[2];  // count = consumer arrivals per item
};

__device__ __forceinline__ void ring_init(ItemRing& r, int consumers) {
  for (int s = 0; s < 2; ++s) {
    mbar_init(&r.full[s], 1);
    mbar_init(&r.empty[s], consumers);
  }
}

// Producer: the CTA's next item (its first is `blockIdx.x`, `claimed` holds a
// counter value taken earlier, or -1 for the first call).
__device__ __forceinline__ Item next_item(const int* ws, int claimed, int count) {
  const int idx = claimed < 0 ? static_cast<int>(blockIdx.x) : claimed + static_cast<int>(gridDim.x);
  return idx < count ? load_item(ws, idx) : kNoItem;
}

__device__ __forceinline__ bool ring_publish(ItemRing& r, uint32_t& st, uint32_t& ph, const Item& item,
                                             volatile int* abort_flag, int* ws, int site) {
  if (!mbar_wait(&r.empty[st], ph ^ 1, abort_flag, ws, site)) return false;
  r.slot[st] = make_int4(item.bh, item.blk, item.n, item.start);
  mbar_arrive(&r.full[st]);
  if (++st == 2) { st = 0; ph ^= 1; }
  return true;
}

// Consumer side: wait for the next slot and copy the item out. A single
// consuming thread releases the slot with ring_release at once; a warp
// releases it once every lane has read it (__syncwarp, then lane 0).
__device__ __forceinline__ bool ring_read(ItemRing& r, uint32_t st, uint32_t ph, Item* item,
                                          volatile int* abort_flag, int* ws, int site) {
  if (!mbar_wait(&r.full[st], ph, abort_flag, ws, site)) return false;
  const int4 v = r.slot[st];  // ordered after the wait by its acquire and memory clobber
  *item = Item{v.x, v.y, v.z, v.w};
  return true;
}

__device__ __forceinline__ void ring_release(ItemRing& r, uint32_t& st, uint32_t& ph, bool arrive) {
  if (arrive) mbar_arrive(&r.empty[st]);
  if (++st == 2) { st = 0; ph ^= 1; }
}

// 1/sqrt(d) for the supported head sizes.
template <int D>
struct Scale;
template <>
struct Scale<64> {
  static constexpr float value = 0.125f;
};
template <>
struct Scale<128> {
  static constexpr float value = 0.08838834764831845f;
};

// The sigmoid of a score, with one MUFU operation. For a score s of sequence
// length n the argument is x = s / sqrt(d) - ln n (Better Models, Faster
// Training: Sigmoid Attention for single-cell Foundation Models, sec. 2A); the
// kernels form y = x log2(e) = s * scale_l2e + neg_log2n in one FMA and take
//
//   u = 2^(-|y|) = e^(-|x|)                      (ex2.approx, relative error ~1e-7)
//   t = -1 + kR2 u + kR3 u^2 + kR4 u^3,  r = 1 + u t  ~  1 / (1 + u) on [0, 1]
//   q = u + (u t) u = u r  ~  sigma(-|x|)
//   sigma(x) = q for x < 0, r for x >= 0;   sigma'(x) = sigma(x) sigma(-x) = q r.
//
// r keeps r(0) = 1 and r'(0) = -1 exactly, so the weights of the far tail (the
// usual case: the bias puts typical weights near 1/n) carry a relative error
// of ~1e-6, and r(1) = 1/2, so sigma(0) = 1/2 and sigma'(0) = 1/4; a minimax
// fit of the other coefficients bounds the relative error of sigma by 9e-4 over
// the whole line (largest near |x| = 1.5), below the bf16 rounding that P
// undergoes next.
//
// The pages' kernel takes sigma from the hardware tanh, 1/2 + tanh(x/2)/2
// (sec. 2C). Measured on B200, that form's error is a few 1e-6 in absolute
// terms, which near 1/n is a relative error of up to 1 % (x in [-12, -8]) and
// which drops every weight below ~1e-7 to zero; with all weights of a row near
// 1/n it shifts O by the same relative amount. The form here costs the same
// single MUFU operation per score, plus FMAs; the choice between q and r runs
// on the integer/logic pipe. A warp whose scores all lie in the far tail takes
// a shorter form without |y|, the polynomial's upper terms or the choice
// (sigmoid32 below).
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kR2 = 0.9339003266f;
constexpr float kR3 = -0.6298789201f;
constexpr float kR4 = 0.1959785935f;

// Two fp32 values in one 64-bit register (first value in the low half), for
// the packed fp32x2 FMAs of sm_100 (one instruction per two values).
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ float2 f2_unpack(uint64_t v) {
  float2 r;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(v));
  return r;
}
__device__ __forceinline__ uint64_t f2_splat(float x) {
  const uint64_t b = __float_as_uint(x);
  return (b << 32) | b;
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// t(u) of two values at once.
__device__ __forceinline__ uint64_t poly_t2(uint64_t u) {
  uint64_t t = f2_fma(f2_splat(kR4), u, f2_splat(kR3));
  t = f2_fma(t, u, f2_splat(kR2));
  return f2_fma(t, u, f2_splat(-1.0f));
}

// The far tail, y < kTailY (sigma < 0.06): with u = 2^y <= 1/16,
// 1 / (1 + u) = 1 - u + u^2 - u^3/(1+u), so q = u (1 - u + u^2) has relative
// error below u^3 <= 2.5e-4 (below 1e-6 once u < 0.01). The kernels evaluate
// it from w = 2^(y + 4) = 16 u as q = w (c + w (-c^2 + c^3 w)), c = 1/16.
constexpr float kTailY = -4.0f;
constexpr float kTailC = 0.0625f;

// sigma of 32 scores of one thread, in place: a[e] holds the fp32 bits of a
// score on entry and of its weight on return; with SLOPE, slope[e] receives
// sigma'. The branch is warp-uniform (every lane of the warp must call this
// together, as the tcgen05 loads that feed it already require): when every
// score of the warp lies in the far tail (the usual case once n is more than
// about a thousand: the bias -ln n puts the typical weight near 1/n), the
// short tail form serves; otherwise the general form. Pairs of columns
// (2e, 2e + 1) go through the packed fp32x2 FMAs. NEG_SLOPE: slope[e]
// receives -sigma' instead (exactly the negation; the tail form then runs its
// polynomial with negated coefficients, which yields -q with no separate sign
// flip, and -sigma' = (-q)^2 + (-q) is one packed FMA), and a[e] receives
// -sigma.
template <bool SLOPE, int N, bool NEG_SLOPE = false>
__device__ __forceinline__ void sigmoid_n(uint32_t (&a)[N], float scale_l2e, float neg_log2n, float* slope,
                                          bool lane_ok = true) {
  static_assert(N == 16 || N == 32, "16 or 32 scores per thread");
  const uint64_t c1 = f2_splat(scale_l2e), c0 = f2_splat(neg_log2n - kTailY);
  uint64_t z[N / 2];  // z = y - kTailY
  uint32_t all = 0xffffffffu;  // AND of the words: bit 31 set iff every z < 0
#pragma unroll
  for (int e = 0; e < N / 2; ++e) {
    z[e] = f2_fma(f2_pack(__uint_as_float(a[2 * e]), __uint_as_float(a[2 * e + 1])), c1, c0);
    all &= static_cast<uint32_t>(z[e]) & static_cast<uint32_t>(z[e] >> 32);
  }
  // Lanes with lane_ok false (rows whose outputs are discarded) take no part
  // in the choice; what they compute is not meaningful.
  if (__all_sync(0xffffffffu, (all >> 31) != 0 || !lane_ok)) {
#pragma unroll
    for (int e = 0; e < N / 2; ++e) {
      const float2 zz = f2_unpack(z[e]);
      const uint64_t w = f2_pack(ex2_approx(zz.x), ex2_approx(zz.y));
      constexpr float sg = NEG_SLOPE ? -1.0f : 1.0f;  // the sign of q that comes out
      uint64_t t = f2_fma(w, f2_splat(sg * kTailC * kTailC * kTailC), f2_splat(-sg * kTailC * kTailC));
      t = f2_fma(t, w, f2_splat(sg * kTailC));
      const uint64_t q = f2_mul(t, w);  // sg * sigma
      const float2 qq = f2_unpack(q);
      if (SLOPE) {
        // NEG_SLOPE: (-q)^2 + (-q) = -(q - q^2) in one packed FMA; otherwise
        // q (1 - q) in two operations, which the dK/dV epilogue schedules
        // better than q - q^2 with a sign flip
        const float2 sl = NEG_SLOPE ? f2_unpack(f2_fma(q, q, q))
                                    : f2_unpack(f2_mul(q, f2_fma(q, f2_splat(-1.0f), f2_splat(1.0f))));
        slope[2 * e] = sl.x;
        slope[2 * e + 1] = sl.y;
      }
      a[2 * e] = __float_as_uint(qq.x);  // sg * sigma
      a[2 * e + 1] = __float_as_uint(qq.y);
    }
  } else {
#pragma unroll
    for (int e = 0; e < N / 2; ++e) {
      const float2 yy = f2_unpack(f2_fma(z[e], f2_splat(1.0f), f2_splat(kTailY)));
      const uint64_t u = f2_pack(ex2_approx(-fabsf(yy.x)), ex2_approx(-fabsf(yy.y)));
      const uint64_t t = poly_t2(u);
      const uint64_t q = f2_fma(f2_mul(t, u), u, u);
      const uint64_t r = f2_fma(t, u, f2_splat(1.0f));
      const float2 qq = f2_unpack(q), rr = f2_unpack(r);
      if (SLOPE) {
        const float2 sl = f2_unpack(NEG_SLOPE ? f2_mul(f2_mul(q, r), f2_splat(-1.0f)) : f2_mul(q, r));
        slope[2 * e] = sl.x;
        slope[2 * e + 1] = sl.y;
      }
      constexpr float sg = NEG_SLOPE ? -1.0f : 1.0f;
      a[2 * e] = __float_as_uint(sg * (yy.x < 0.0f ? qq.x : rr.x));
      a[2 * e + 1] = __float_as_uint(sg * (yy.y < 0.0f ? qq.y : rr.y));
    }
  }
}

template <bool SLOPE>
__device__ __forceinline__ void sigmoid32(uint32_t (&a)[32], float scale_l2e, float neg_log2n, float* slope,
                                          bool lane_ok = true) {
  sigmoid_n<SLOPE, 32>(a, scale_l2e, neg_log2n, slope, lane_ok);
}

// Scores that must not count: the columns at or past `valid` (keys beyond
// the sequence) and every column of a row that is not a valid token. Set to
// -inf, their weight and its derivative come out exactly 0 on either form,
// and they take no part in the warp's choice of form, so values in padded
// rows never change the bits of a valid output.
template <int N>
__device__ __forceinline__ void mask_scores(uint32_t (&a)[N], int valid, bool row_ok) {
  if (valid >= N && row_ok) return;
#pragma unroll
  for (int e = 0; e < N; ++e)
    if (!row_ok || e >= valid) a[e] = 0xff800000u;
}

// sigma (and sigma') of one score, as the kernels compute it (the diagnostic
// entry point; its warp takes the tail form only when all 32 lanes' scores are
// in the far tail).
__device__ __forceinline__ float sigmoid_score(float s, float scale_l2e, float neg_log2n, float* slope) {
  uint32_t a[32];
  float sl[32];
#pragma unroll
  for (int e = 0; e < 32; ++e) a[e] = __float_as_uint(s);
  sigmoid_n<true, 32, true>(a, scale_l2e, neg_log2n, sl);  // the dQ kernel's form
  *slope = -sl[0];
  return -__uint_as_float(a[0]);
}

// Zero one unit of the output rows that no work item covers: rows
// [cover, out_rows) of slice u / parts (cover: the rows the call's items
// write) are cut into `parts` interleaved shares of 16-byte chunks, and this
// warp writes share u % parts of out0 (and out1).
__device__ __forceinline__ void zero_fill_unit(const int* lengths, const FillGeom& g, int parts, long long u, int lane,
                                               void* out0, void* out1) {
  const int slice = static_cast<int>(u / parts);
  const int part = static_cast<int>(u % parts);
  const int cover = g.cover(load_len(lengths, slice / g.H, g.L));
  const long long nchunks = static_cast<long long>(g.out_rows - cover) * g.chunks_per_row;
  const size_t base = (static_cast<size_t>(slice) * g.out_rows + cover) * g.chunks_per_row;
  uint4* p0 = reinterpret_cast<uint4*>(out0) + base;
  uint4* p1 = out1 ? reinterpret_cast<uint4*>(out1) + base : nullptr;
  for (long long c = static_cast<long long>(part) * 32 + lane; c < nchunks; c += static_cast<long long>(parts) * 32) {
    p0[c] = make_uint4(0, 0, 0, 0);
    if (p1) p1[c] = make_uint4(0, 0, 0, 0);
  }
}

// The same rows cut into `parts` consecutive shares instead (the dQ kernel's
// fill, whose units go either to bulk copies or to warps): unit u covers the
// 16-byte chunks [begin, end) counted from 16-byte chunk `base` of the output.
struct FillRange {
  size_t base;
  long long begin, end;
};

__device__ __forceinline__ FillRange zero_fill_range(const int* lengths, const FillGeom& g, int parts, long long u) {
  const int slice = static_cast<int>(u / parts);
  const int part = static_cast<int>(u % parts);
  const int cover = g.cover(load_len(lengths, slice / g.H, g.L));
  const long long nchunks = static_cast<long long>(g.out_rows - cover) * g.chunks_per_row;
  const long long share = (nchunks + parts - 1) / parts;
  FillRange f;
  f.base = (static_cast<size_t>(slice) * g.out_rows + cover) * g.chunks_per_row;
  f.begin = min(nchunks, part * share);
  f.end = min(nchunks, f.begin + share);
  return f;
}

// One warp writes the zeros of a consecutive-share unit.
__device__ __forceinline__ void zero_fill_range_warp(const FillRange& f, int lane, void* out) {
  uint4* p = reinterpret_cast<uint4*>(out) + f.base;
  for (long long c = f.begin + lane; c < f.end; c += 32) p[c] = make_uint4(0, 0, 0, 0);
}

// Shares per slice for the zero fill: enough units to spread over the SMs.
inline int zero_fill_parts(long long slices, int num_sms) {
  return static_cast<int>(std::max<long long>(1, std::min<long long>(64, (4LL * num_sms + slices - 1) / slices)));
}

// Store 64 bytes (one row's 32 bf16 values, packed in pairs) at dst, which is
// 16-byte aligned. An epilogue lane owns one row, so a warp's store touches 32
// rows; 32-byte stores halve the number of such instructions when dst is
// 32-byte aligned (warp-uniform: row strides are multiples of 32 bytes).
__device__ __forceinline__ void store_row64B(void* dst, const uint32_t (&w)[16]) {
  if ((reinterpret_cast<uintptr_t>(dst) & 31u) == 0) {
#pragma unroll
    for (int h = 0; h < 2; ++h)
      asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(
                       reinterpret_cast<uint8_t*>(dst) + 32 * h),
                   "r"(w[8 * h]), "r"(w[8 * h + 1]), "r"(w[8 * h + 2]), "r"(w[8 * h + 3]), "r"(w[8 * h + 4]),
                   "r"(w[8 * h + 5]), "r"(w[8 * h + 6]), "r"(w[8 * h + 7])
                   : "memory");
  } else {
    uint4* p = reinterpret_cast<uint4*>(dst);
#pragma unroll
    for (int q = 0; q < 4; ++q) p[q] = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
  }
}

// Store NW 32-bit words (32, 64 or 128 bytes of one row) at dst, 16-byte
// aligned; 32-byte stores when dst is 32-byte aligned (warp-uniform).
template <int NW>
__device__ __forceinline__ void store_words(void* dst, const uint32_t (&w)[NW]) {
  static_assert(NW % 8 == 0, "whole 32-byte pieces");
  if ((reinterpret_cast<uintptr_t>(dst) & 31u) == 0) {
#pragma unroll
    for (int h = 0; h < NW / 8; ++h)
      asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(
                       reinterpret_cast<uint8_t*>(dst) + 32 * h),
                   "r"(w[8 * h]), "r"(w[8 * h + 1]), "r"(w[8 * h + 2]), "r"(w[8 * h + 3]), "r"(w[8 * h + 4]),
                   "r"(w[8 * h + 5]), "r"(w[8 * h + 6]), "r"(w[8 * h + 7])
                   : "memory");
  } else {
    uint4* p = reinterpret_cast<uint4*>(dst);
#pragma unroll
    for (int q = 0; q < NW / 4; ++q) p[q] = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
  }
}

// Convert 32 fp32 accumulator values (times `mul`) to bf16 and store them.
__device__ __forceinline__ void store_row32(__nv_bfloat16* dst, const uint32_t (&v)[32], float mul) {
  uint32_t w[16];
#pragma unroll
  for (int e = 0; e < 16; ++e)
    w[e] = pack_bf16x2(__uint_as_float(v[2 * e]) * mul, __uint_as_float(v[2 * e + 1]) * mul);
  store_row64B(dst, w);
}

__device__ __forceinline__ void store_zero32(__nv_bfloat16* dst) {
  uint32_t w[16];
#pragma unroll
  for (int e = 0; e < 16; ++e) w[e] = 0u;
  store_row64B(dst, w);
}

// A set-up step (a kernel attribute) run once per device, safely across host
// threads: the first caller on a device runs it, later callers get its result.
struct PerDeviceOnce {
  static constexpr int kDevices = 64;
  std::once_flag flag[kDevices];
  cudaError_t err[kDevices] = {};
  template <typename F>
  cudaError_t run(F&& setup) {
    int dev = 0;
    const cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kDevices) return cudaErrorInvalidDevice;
    std::call_once(flag[dev], [&] { err[dev] = setup(); });
    return err[dev];
  }
};

// Store 32 fp32 values (one row's 32 columns, 128 bytes) at dst, 16-byte
// aligned; 32-byte stores when dst is 32-byte aligned (warp-uniform).
__device__ __forceinline__ void store_row_f32(float* dst, const uint32_t (&v)[32]) {
  if ((reinterpret_cast<uintptr_t>(dst) & 31u) == 0) {
#pragma unroll
    for (int h = 0; h < 4; ++h)
      asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(dst + 8 * h), "r"(v[8 * h]),
                   "r"(v[8 * h + 1]), "r"(v[8 * h + 2]), "r"(v[8 * h + 3]), "r"(v[8 * h + 4]), "r"(v[8 * h + 5]),
                   "r"(v[8 * h + 6]), "r"(v[8 * h + 7])
                   : "memory");
  } else {
    uint4* p = reinterpret_cast<uint4*>(dst);
#pragma unroll
    for (int q = 0; q < 8; ++q) p[q] = make_uint4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
  }
}

// An output row chunk of 32 columns at element offset `off` of `out`: bf16
// (rounded, times `mul`) or, for the fp32 partial sums of a key-range call,
// the fp32 values themselves (times `mul`). `zero` writes zeros instead.
template <bool F32OUT>
__device__ __forceinline__ void store_out32(void* out, size_t off, const uint32_t (&v)[32], float mul, bool zero) {
  if constexpr (F32OUT) {
    uint32_t w[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) w[e] = zero ? 0u : __float_as_uint(__uint_as_float(v[e]) * mul);
    store_row_f32(static_cast<float*>(out) + off, w);
  } else {
    __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(out) + off;
    if (zero) store_zero32(dst);
    else store_row32(dst, v, mul);
  }
}

template <bool F32OUT>
__device__ __forceinline__ void store_zero_out32(void* out, size_t off) {
  if constexpr (F32OUT) {
    uint32_t w[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) w[e] = 0u;
    store_row_f32(static_cast<float*>(out) + off, w);
  } else {
    store_zero32(static_cast<__nv_bfloat16*>(out) + off);
  }
}

// Launch `kernel` so that it may start while the previous kernel in `stream` is
// still running (programmatic stream serialization). The kernel calls
// grid_dep_wait() before it touches anything that earlier kernel writes.
template <typename... Params, typename... Args>
inline cudaError_t launch_programmatic(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem,
                                       cudaStream_t stream, Args&&... args) {
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

}  // namespace sigattn
