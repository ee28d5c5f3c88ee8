// plan.cu -- the ragged tile scheduler and padded-row zero fill.
//
// "Native padding support": blocks that hold only padding are skipped on both
// the query and the key side (Better Models, Faster Training: Sigmoid
// Attention for single-cell Foundation Models, sec. 2C). Here that becomes a
// work list built on the device from the per-sequence valid lengths, so the
// host never has to read the lengths back:
//
//   * one work item per (b, h, row block) whose first row is < n_b; the
//     compute kernels walk column blocks only up to ceil(n_b / block width);
//   * sequences are ordered longest first (stable in b), and a persistent
//     compute grid takes items round-robin, which spreads the long items over
//     all SMs first (longest-processing-time-first order);
//   * rows of the outputs that no item covers (rows >= ceil(n_b/rows)*rows)
//     are written as exact zeros: after the forward kernel by fill_kernel, a
//     one-warp-per-CTA kernel launched with a programmatic edge, so that it
//     runs on the registers and warps the persistent compute CTA leaves free
//     and its HBM writes overlap the compute-bound kernel; the backward
//     kernels, whose CTAs take all of an SM's registers, zero their own: their
//     warps without a role from the start and every other warp once its role
//     is done claim fill units from a counter in the workspace header (at
//     d = 64 the dQ kernel's producer also issues bulk copies from a block of
//     zeros in shared memory, one fill unit per work item).
//   * a call over a key range (a contiguous range of key positions of every
//     sequence) enumerates the rows that have work: for the forward and dQ all
//     query rows of a sequence with a valid key in the range, for dK/dV the
//     range's valid keys; the items are ordered by their column counts.
#include <algorithm>
#include <numeric>
#include <vector>

#include "common.cuh"

namespace sigattn {

// Sequence lengths come either from `lengths` (padded layout) or, when `cu`
// is given, from cumulative offsets: sequence b holds packed tokens
// [cu[b], cu[b+1]), which must lie inside [0, total_tokens]. A sequence that breaks
// its bounds gets no work items and raises SIGATTN_ERR_INVALID_ARG.
// One CTA per work list: CTA i builds list `lists[i]` (a whole-backward call
// builds the dQ and the dK/dV lists at once); length errors go to `err`.
struct PlanLists {
  PlanRegion list[2];
};

__global__ void __launch_bounds__(1024) prep_kernel(const int* __restrict__ lengths, const int* __restrict__ cu,
                                                    int total_tokens, int B, int H, int L, PlanLists lists,
                                                    int* __restrict__ err) {
  // The compute kernel that follows may set itself up meanwhile; it waits
  // for this grid before it reads the plan.
  grid_dep_launch();
  const PlanRegion region = lists.list[blockIdx.x];
  const int kind = region.kind;
  const KeyRange kr = region.kr;
  int* __restrict__ ws = region.ws;
  extern __shared__ int smem_plan[];
  const int tid = threadIdx.x;
  const int rows = item_rows(kind);
  int* s_len = smem_plan;            // [B]
  int* s_order = smem_plan + B;      // [B]
  int* s_off = smem_plan + 2 * B;    // [B + 1]
  int* s_start = smem_plan + 3 * B + 1;  // [B]
  int* s_key = smem_plan + 4 * B + 1;    // [B] columns per item (the sort key)
  for (int b = tid; b < B; b += blockDim.x) {
    int n, start = 0;
    bool bad;
    if (cu != nullptr) {
      start = __ldg(cu + b);
      const int end = __ldg(cu + b + 1);
      n = end - start;
      bad = start < 0 || end < start || end > total_tokens || n > L;
    } else {
      n = __ldg(lengths + b);
      bad = n < 0 || n > L;
    }
    if (bad) {
      atomicCAS(err + kHdrError, 0, 1 /* SIGATTN_ERR_INVALID_ARG */);
      atomicExch(err + kHdrErrorSite, -(b + 1));
    }
    s_len[b] = bad ? 0 : n;
    s_start[b] = bad ? 0 : start;
    s_key[b] = work_rows(kind, s_len[b], kr) > 0 ? work_cols(kind, s_len[b], kr) : 0;
  }
  __syncthreads();
  // Rank of each sequence in the longest-first order of its items' column
  // counts (ties keep batch order).
  for (int b = tid; b < B; b += blockDim.x) {
    const int nb = s_key[b];
    int rank = 0;
    for (int o = 0; o < B; ++o) {
      const int no = s_key[o];
      rank += (no > nb) || (no == nb && o < b);
    }
    s_order[rank] = b;
  }
  __syncthreads();
  if (tid == 0) s_off[0] = 0;
  for (int s = tid; s < B; s += blockDim.x) s_off[s + 1] = H * ceil_div(work_rows(kind, s_len[s_order[s]], kr), rows);
  __syncthreads();
  // Inclusive scan of s_off[1..B] by warp 0, 32 entries at a time.
  if (tid < 32) {
    int carry = 0;
    for (int base = 0; base < B; base += 32) {
      const int i = base + tid;
      int v = (i < B) ? s_off[i + 1] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, v, o);
        if (tid >= o) v += u;
      }
      v += carry;
      if (i < B) s_off[i + 1] = v;
      carry = __shfl_sync(0xffffffffu, v, 31);
    }
  }
  __syncthreads();
  const int total = s_off[B];
  if (tid == 0) {
    ws[kHdrCount] = total;
    ws[kHdrNext] = 0;  // the compute kernel's claim counter
    ws[kHdrFill] = 0;  // the dQ kernel's zero-fill claim counter
  }
  // Each thread writes one contiguous run of the list: item i of sequence
  // rank s is (b, h, blk) with (h, blk) = divmod(i - s_off[s], row blocks of
  // b); the first item of the run is located by a binary search, the others
  // by counting on, so the run costs no search or division per item.
  int4* items = reinterpret_cast<int4*>(ws + kHeaderWords);
  const int per = ceil_div(total, static_cast<int>(blockDim.x));
  const int first = tid * per, end = min(total, first + per);
  if (first < end) {
    int lo = 0, hi = B - 1;  // the last s with s_off[s] <= first (a sequence with items)
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_off[mid] <= first) lo = mid; else hi = mid - 1;
    }
    int b = s_order[lo];
    int nblk = ceil_div(work_rows(kind, s_len[b], kr), rows);
    int h = (first - s_off[lo]) / nblk, blk = (first - s_off[lo]) % nblk;
    for (int i = first; i < end; ++i) {
      items[i] = make_int4(b * H + h, blk, s_len[b], s_start[b]);
      if (++blk < nblk) continue;
      blk = 0;
      if (++h < H || i + 1 == end) continue;
      h = 0;  // on to the next sequence with items
      do ++lo; while (s_off[lo + 1] == s_off[lo]);
      b = s_order[lo];
      nblk = ceil_div(work_rows(kind, s_len[b], kr), rows);
    }
  }
}

// The plan kernel's shared memory (5 B + 1 ints) may exceed the default
// 48 KB for large batches: raise its limit once per device.
static cudaError_t prep_setup() {
  static PerDeviceOnce attr;
  return attr.run([] {
    return cudaFuncSetAttribute(prep_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (5 * kMaxBatch + 1) * static_cast<int>(sizeof(int)));
  });
}

cudaError_t launch_prep(const int* lengths, const int* cu, int total, int B, int H, int L, int kind, KeyRange kr,
                        int* ws, cudaStream_t stream) {
  const cudaError_t e = prep_setup();
  if (e != cudaSuccess) return e;
  const int smem = (5 * B + 1) * static_cast<int>(sizeof(int));
  const int threads = B <= 256 ? 256 : 1024;
  PlanLists lists{{PlanRegion{kind, kr, ws}, PlanRegion{kind, kr, ws}}};
  prep_kernel<<<1, threads, smem, stream>>>(lengths, cu, total, B, H, L, lists, ws);
  return cudaGetLastError();
}

// The dQ and dK/dV lists of a whole-backward call (whole sequences, padded
// layout from `lengths` or packed from `cu` as in launch_prep) in one launch:
// the dQ list in ws_dq, the dK/dV list in ws_dkdv; errors go to ws_dq's header.
cudaError_t launch_prep_bwd(const int* lengths, const int* cu, int total, int B, int H, int L, int* ws_dq,
                            int* ws_dkdv, cudaStream_t stream) {
  const cudaError_t e = prep_setup();
  if (e != cudaSuccess) return e;
  const int smem = (5 * B + 1) * static_cast<int>(sizeof(int));
  const int threads = B <= 256 ? 256 : 1024;
  const KeyRange all{0, L};
  PlanLists lists{{PlanRegion{kKindDq, all, ws_dq}, PlanRegion{kKindDkdv, all, ws_dkdv}}};
  prep_kernel<<<2, threads, smem, stream>>>(lengths, cu, total, B, H, L, lists, ws_dq);
  return cudaGetLastError();
}

// Zero the output rows that no work item covers, rows [ceil(n_b/rows)*rows, L)
// of every (b, h) slice, in out0 (and out1). One warp per CTA: it fits beside
// a persistent compute CTA in what that leaves of the SM's registers. Each
// slice is cut into `parts` interleaved shares so that the CTAs stay balanced
// when B*H is small. The final wait keeps the stream order: this grid (and so
// the call) completes only after the compute kernel before it.
__global__ void __launch_bounds__(32) fill_kernel(const int* __restrict__ lengths, int B, FillGeom g, int parts,
                                                  void* out0, void* out1) {
  const long long units = static_cast<long long>(B) * g.H * parts;
  for (long long u = blockIdx.x; u < units; u += gridDim.x) zero_fill_unit(lengths, g, parts, u, threadIdx.x, out0, out1);
  grid_dep_wait();
}

// The fill overlaps the forward kernel (the backward kernels zero their own
// uncovered rows, see bwd.cu). elem_bytes is 2 for bf16 outputs and 4 for the
// fp32 partial sums of a key-range forward.
cudaError_t launch_fill(const int* lengths, int B, int H, int L, int d, int kind, KeyRange kr, int elem_bytes,
                        void* out0, void* out1, int num_sms, cudaStream_t stream) {
  const int parts = zero_fill_parts(static_cast<long long>(B) * H, num_sms);
  const int grid = std::max(1, num_sms);
  const FillGeom g{H, L, kind == kKindDkdv ? kr.count : L, d * elem_bytes / 16, kind, item_rows(kind), kr};
  return launch_programmatic(fill_kernel, dim3(grid), dim3(32), 0, stream, lengths, B, g, parts, out0, out1);
}

// Diagnostic: one warp waits, with a bounded wait, on an mbarrier that nothing
// arrives on. The wait must give up after `limit_ns` and record the timeout in
// the workspace header exactly as a compute kernel's wait would (site 901).
__global__ void selftest_timeout_kernel(int* ws, unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag, ws, 901, limit_ns);
  __syncthreads();
}

cudaError_t launch_selftest_timeout(int* ws, unsigned long long limit_ns, cudaStream_t stream) {
  selftest_timeout_kernel<<<1, 32, 0, stream>>>(ws, limit_ns);
  return cudaGetLastError();
}

// Diagnostic: the sigmoid of scores exactly as the compute kernels evaluate it
// (sigmoid_score with the kernels' constants for head size D and length n),
// and its derivative as the backward kernels use it.
// Each warp takes 32 consecutive scores per step (the sigmoid's branch is
// warp-uniform, so all 32 lanes stay in the loop; lanes past `count` compute a
// dummy score and store nothing).
template <int D>
__global__ void eval_sigmoid_kernel(const float* __restrict__ s, float* __restrict__ p, float* __restrict__ slope,
                                    int count, int n) {
  const float scale_l2e = Scale<D>::value * kLog2e;
  const float neg_log2n = -__log2f(static_cast<float>(n));
  const int lane = threadIdx.x & 31;
  const long long warps = static_cast<long long>(gridDim.x) * (blockDim.x >> 5);
  for (long long base = (blockIdx.x * static_cast<long long>(blockDim.x >> 5) + (threadIdx.x >> 5)) * 32; base < count;
       base += warps * 32) {
    const long long i = base + lane;
    float dp;
    const float v = sigmoid_score(i < count ? s[i] : 0.0f, scale_l2e, neg_log2n, &dp);
    if (i < count) {
      p[i] = v;
      slope[i] = dp;
    }
  }
}

cudaError_t launch_eval_sigmoid(const float* s, float* p, float* slope, int count, int d, int n, int num_sms,
                                cudaStream_t stream) {
  const int grid = std::max(1, std::min(4 * num_sms, ceil_div(count, 256)));
  if (d == 64)
    eval_sigmoid_kernel<64><<<grid, 256, 0, stream>>>(s, p, slope, count, n);
  else
    eval_sigmoid_kernel<128><<<grid, 256, 0, stream>>>(s, p, slope, count, n);
  return cudaGetLastError();
}

// fp32 -> bf16 (round to nearest even), eight values per thread and step:
// the last step of a key-sharded call, after its fp32 partial sums were added.
__global__ void cast_bf16_kernel(const float4* __restrict__ in, uint4* __restrict__ out, long long n8) {
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n8;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const float4 a = in[2 * i], b = in[2 * i + 1];
    out[i] = make_uint4(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w), pack_bf16x2(b.x, b.y), pack_bf16x2(b.z, b.w));
  }
}

cudaError_t launch_cast_bf16(const float* in, void* out, long long count, int num_sms, cudaStream_t stream) {
  const long long n8 = count / 8;
  const int grid = static_cast<int>(std::max<long long>(1, std::min<long long>(8LL * num_sms, (n8 + 255) / 256)));
  cast_bf16_kernel<<<grid, 256, 0, stream>>>(reinterpret_cast<const float4*>(in), static_cast<uint4*>(out), n8);
  return cudaGetLastError();
}

// Host restatement of the same schedule (used by the host-side tests and for
// debugging): items in the order the device plan writes them.
int plan_host(const int* lengths, int B, int H, int L, int kind, int* out, int cap) {
  const int rows = item_rows(kind);
  std::vector<int> len(B), order(B);
  for (int b = 0; b < B; ++b) len[b] = (lengths[b] < 0 || lengths[b] > L) ? 0 : lengths[b];
  std::iota(order.begin(), order.end(), 0);
  std::stable_sort(order.begin(), order.end(), [&](int a, int b) { return len[a] > len[b]; });
  int count = 0;
  for (int s = 0; s < B; ++s) {
    const int b = order[s];
    const int nblk = ceil_div(len[b], rows);
    for (int h = 0; h < H; ++h)
      for (int m = 0; m < nblk; ++m) {
        if (count < cap) {
          out[2 * count] = b * H + h;
          out[2 * count + 1] = m;
        }
        ++count;
      }
  }
  return count;
}

}  // namespace sigattn
