// Expert parallelism: the data movement around the all-to-all exchanges.
//
// Each rank owns El consecutive experts.  A source rank sorts its routed rows
// by (expert, token, slot) in compact order (moe_ep_dispatch_pack), so the
// rows for a destination rank form one contiguous range; the exchange
// delivers them source-major: source s's rows for local expert 0, 1, ...,
// then source s + 1's.  On the destination:
//   * k_ep_tables turns the [G][El] row counts into the local group offsets
//     and, per (source, expert) pair, where its rows start in the received
//     buffer, in the padded grouped layout and in compact local order;
//   * k_ep_arrange places the received rows into the padded grouped layout
//     the grouped GEMMs read (expert-major, source-major within an expert;
//     scales from row-major to K-step-major; padding rows zeroed);
//   * k_ep_return puts the compact D rows back into received order, which is
//     the order the reverse exchange returns them in, and on the source the
//     concatenated returns are its compact sorted rows again.
// The exchanges themselves are NCCL all-to-alls outside the library.
#include "common.cuh"
#include "internal.h"

namespace nvfp4moe {

namespace {

constexpr int kTableThreads = 1024;

// One block.  counts [G][El] (int32, source-major).  Writes:
//   offsets[El+1], padded[El+1]        local groups (padded to 128 rows)
//   tab[0*P + s*El + e]  recv_start:   first received row of pair (s, e)
//   tab[1*P + s*El + e]  pad_start:    its first padded row
//   tab[2*P + s*El + e]  cmp_start:    its first compact local row
// with P = G * El <= 1024.
__global__ void __launch_bounds__(kTableThreads) k_ep_tables(const int32_t *__restrict__ counts, int G, int El,
                                                              int32_t *offsets, int32_t *padded, int32_t *tab,
                                                              int *err) {
  __shared__ int32_t s_flat[kTableThreads];
  __shared__ int32_t s_n[kTableThreads], s_np[kTableThreads];
  const int P = G * El;
  const int t = threadIdx.x;
  // received order is source-major: exclusive scan of the flat counts
  int32_t c = 0;
  if (t < P) {
    c = __ldg(counts + t);
    if (c < 0) {
      set_device_error(err, kDevBadInput, t);
      c = 0;
    }
  }
  s_flat[t] = c;
  // per local expert: rows from every source, and the padded size
  int32_t n = 0;
  if (t < El)
    for (int s = 0; s < G; ++s) n += max(__ldg(counts + s * El + t), 0);
  s_n[t] = t < El ? n : 0;
  s_np[t] = t < El ? (n + 127) / 128 * 128 : 0;
  __syncthreads();
  // Hillis-Steele inclusive scans (1024 entries, one block)
  for (int o = 1; o < kTableThreads; o <<= 1) {
    const int32_t a = t >= o ? s_flat[t - o] : 0;
    const int32_t b = t >= o ? s_n[t - o] : 0;
    const int32_t d = t >= o ? s_np[t - o] : 0;
    __syncthreads();
    s_flat[t] += a;
    s_n[t] += b;
    s_np[t] += d;
    __syncthreads();
  }
  if (t == 0) {
    offsets[0] = 0;
    padded[0] = 0;
  }
  if (t < El) {
    offsets[t + 1] = s_n[t];
    padded[t + 1] = s_np[t];
  }
  if (t < P) {
    const int s = t / El, e = t - s * El;
    int32_t before = 0;                       // rows of expert e from sources < s
    for (int q = 0; q < s; ++q) before += max(__ldg(counts + q * El + e), 0);
    const int32_t off_e = e == 0 ? 0 : s_n[e - 1];
    const int32_t pad_e = e == 0 ? 0 : s_np[e - 1];
    tab[t] = s_flat[t] - c;                   // exclusive
    tab[P + t] = pad_e + before;
    tab[2 * P + t] = off_e + before;
  }
}

// The pair (s, e) whose received range holds row i < rows_recv: the last
// pair with recv_start <= i (recv_start is non-decreasing; an empty pair
// shares its start with the next one, so the last such pair has rows).
__device__ __forceinline__ int pair_of(const int32_t *recv_start, int P, int64_t i) {
  int lo = 0, hi = P;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if ((int64_t)__ldg(recv_start + mid) <= i) lo = mid; else hi = mid;
  }
  return lo;
}

constexpr int kRowWarps = 8;

// One warp per padded row p of the local grouped layout.
__global__ void __launch_bounds__(kRowWarps * 32) k_ep_arrange(const EpArrangeParams a) {
  const int lane = threadIdx.x & 31;
  const int64_t p = (int64_t)blockIdx.x * kRowWarps + (threadIdx.x >> 5);
  int64_t used = __ldg(a.padded + a.El);
  if (used > a.rows_cap) used = a.rows_cap;
  if (p >= used) return;
  int lo = 0, hi = a.El;                      // the local expert of row p
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if ((int64_t)__ldg(a.padded + mid) <= p) lo = mid; else hi = mid;
  }
  const int e = lo;
  const int64_t rel = p - __ldg(a.padded + e);
  const int64_t n_e = (int64_t)__ldg(a.offsets + e + 1) - __ldg(a.offsets + e);
  const int P = a.G * a.El;
  const int64_t qv = a.H / 32;                // uint4 of codes per row
  const int64_t ksteps = a.H / 256;
  uint4 *qd = reinterpret_cast<uint4 *>(a.q_a) + p * qv;
  const uint4 z = make_uint4(0, 0, 0, 0);
  if (rel >= n_e) {                           // padding row: zero codes, scales and S_dec
    for (int64_t c = lane; c < qv; c += 32) qd[c] = z;
    for (int64_t kt = lane; kt < ksteps; kt += 32)
      *reinterpret_cast<uint4 *>(a.sf_a + (kt * a.rows_cap + p) * 16) = z;
    if (lane == 0) a.sdec_a[p] = 0.0f;
    return;
  }
  // the source of this row: pad_start[s][e] <= p, last such s with rows
  const int32_t *pad_start = a.tab + P;
  int s = 0;
  for (int q = 1; q < a.G; ++q)
    if ((int64_t)__ldg(pad_start + q * a.El + e) <= p && __ldg(a.counts + q * a.El + e) > 0) s = q;
  const int64_t i = (int64_t)__ldg(a.tab + s * a.El + e) + (p - __ldg(pad_start + s * a.El + e));
  if (i < 0 || i >= a.rows_recv) {
    if (lane == 0) set_device_error(a.err, kDevBadInput, (int)p);
    return;
  }
  const uint4 *qs = reinterpret_cast<const uint4 *>(a.q_recv) + i * qv;
  for (int64_t c = lane; c < qv; c += 32) qd[c] = __ldg(qs + c);
  // scales: row-major [H/16] per row -> K-step-major [H/256][rows_cap][16]
  const uint4 *ss = reinterpret_cast<const uint4 *>(a.sf_recv + i * (a.H / 16));
  for (int64_t kt = lane; kt < ksteps; kt += 32)
    *reinterpret_cast<uint4 *>(a.sf_a + (kt * a.rows_cap + p) * 16) = __ldg(ss + kt);
  if (lane == 0) a.sdec_a[p] = __ldg(a.sdec_recv + i);
}

// One warp per received row i: d_send[i] = d[compact local row of i].
__global__ void __launch_bounds__(kRowWarps * 32) k_ep_return(const void *__restrict__ d, const int32_t *tab, int P,
                                                               int64_t rows_recv, int64_t H, void *__restrict__ d_send,
                                                               int *err) {
  const int lane = threadIdx.x & 31;
  const int64_t i = (int64_t)blockIdx.x * kRowWarps + (threadIdx.x >> 5);
  if (i >= rows_recv) return;
  const int q = pair_of(tab, P, i);
  const int64_t c = (int64_t)__ldg(tab + 2 * P + q) + (i - __ldg(tab + q));
  if (c < 0 || c >= rows_recv) {
    if (lane == 0) set_device_error(err, kDevBadInput, (int)i);
    return;
  }
  const int64_t hv = H / 8;                   // uint4 of BF16 per row
  const uint4 *src = static_cast<const uint4 *>(d) + c * hv;
  uint4 *dst = static_cast<uint4 *>(d_send) + i * hv;
  for (int64_t x = lane; x < hv; x += 32) dst[x] = __ldg(src + x);
}

}  // namespace

cudaError_t launch_ep_tables(const int32_t *counts, int G, int El, int32_t *offsets, int32_t *padded, int32_t *tab,
                             int *err, cudaStream_t s) {
  if (G < 1 || El < 1 || G * El > kTableThreads) return cudaErrorInvalidValue;
  k_ep_tables<<<1, kTableThreads, 0, s>>>(counts, G, El, offsets, padded, tab, err);
  return cudaGetLastError();
}

cudaError_t launch_ep_arrange(const EpArrangeParams &a, cudaStream_t s) {
  if (a.rows_cap <= 0) return cudaSuccess;
  k_ep_arrange<<<(unsigned)((a.rows_cap + kRowWarps - 1) / kRowWarps), kRowWarps * 32, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_ep_return(const void *d, const int32_t *tab, int P, int64_t rows_recv, int64_t H, void *d_send,
                             int *err, cudaStream_t s) {
  if (rows_recv <= 0) return cudaSuccess;
  k_ep_return<<<(unsigned)((rows_recv + kRowWarps - 1) / kRowWarps), kRowWarps * 32, 0, s>>>(d, tab, P, rows_recv, H,
                                                                                          d_send, err);
  return cudaGetLastError();
}

}  // namespace nvfp4moe
