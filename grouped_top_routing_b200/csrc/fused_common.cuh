// Helpers of the fused decode kernel (decode_fused.cu): bounded waits, the
// grid barrier, even splits of a phase over the CTAs, and the counting of
// output rows. Every wait is bounded by DecodeArgs::wait_ns (globaltimer;
// moe_options.wait_limit_ns, 2 s by default): one that runs out records
// MOE_ERR_TIMEOUT in the workspace and returns false.
#pragma once

#include "decode_fused.cuh"
#include "mbarrier.cuh"

namespace moe {
namespace fused {

constexpr int kMaxSlots = 32;  // T * k; also the number of expert counters at the start of DecodeArgs::sync
// Every poll loop sleeps this long between polls, so a waiting warp (a
// producer above all, which shares a scheduler with consumer warps) leaves
// the issue slots to the warps doing the work.
constexpr unsigned kBackoffNs = 32;

struct Range {
  int lo, n;
};

// Contiguous share b of G of `total` items.
__host__ __device__ __forceinline__ Range split(int total, int b, int G) {
  const int lo = (int)((int64_t)total * b / G), hi = (int)((int64_t)total * (b + 1) / G);
  return {lo, hi - lo};
}

__device__ __forceinline__ int ld_acquire(const int32_t* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void red_release_add(int32_t* p, int v) {
  asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ float4 ldcg4(const float* p) { return __ldcg(reinterpret_cast<const float4*>(p)); }

// Bounded wait for the phase of `bar` with the given parity, by every lane of
// the warp; false (in every lane) after recording a timeout.
__device__ inline bool warp_wait_phase(uint64_t* bar, uint32_t parity, WsHeader* hdr, int site, uint64_t limit) {
  int ok = 1;
  if (!mbar_try_wait(bar, parity)) {
    const uint64_t t0 = globaltimer();
    while (!mbar_try_wait(bar, parity)) {
      if (globaltimer() - t0 > limit) {
        ok = 0;
        break;
      }
      __nanosleep(kBackoffNs);
    }
  }
  ok = __all_sync(0xffffffffu, ok);
  if (!ok && (threadIdx.x & 31) == 0) record_error(hdr, MOE_ERR_TIMEOUT, site);
  return ok != 0;
}

// Bounded wait until the producer tagged slot `tag` with stream index v.
__device__ inline bool warp_wait_tag(volatile uint32_t* tag, uint32_t v, WsHeader* hdr, int site, uint64_t limit) {
  int ok = 1;
  if (*tag != v) {
    const uint64_t t0 = globaltimer();
    while (*tag != v) {
      if (globaltimer() - t0 > limit) {
        ok = 0;
        break;
      }
      __nanosleep(kBackoffNs);
    }
  }
  ok = __all_sync(0xffffffffu, ok);
  if (!ok && (threadIdx.x & 31) == 0) record_error(hdr, MOE_ERR_TIMEOUT, site);
  return ok != 0;
}

// Single-thread bounded wait (producer side).
__device__ inline bool thread_wait_phase(uint64_t* bar, uint32_t parity, WsHeader* hdr, int site, uint64_t limit) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer() - t0 > limit) {
      if (hdr != nullptr) record_error(hdr, MOE_ERR_TIMEOUT, site);
      return false;
    }
    __nanosleep(kBackoffNs);
  }
  return true;
}

// Lane 0 waits (bounded) until *ctr >= target; the whole warp then sees every
// write released before the increments. False after recording a timeout.
__device__ inline bool warp_wait_count(const int32_t* ctr, int target, WsHeader* hdr, int site, uint64_t limit) {
  int ok = 1;
  if ((threadIdx.x & 31) == 0 && ld_acquire(ctr) < target) {
    const uint64_t t0 = globaltimer();
    while (ld_acquire(ctr) < target) {
      if (globaltimer() - t0 > limit) {
        record_error(hdr, MOE_ERR_TIMEOUT, site);
        ok = 0;
        break;
      }
      __nanosleep(kBackoffNs);
    }
  }
  ok = __shfl_sync(0xffffffffu, ok, 0);
  __syncwarp();
  return ok != 0;
}

__device__ __forceinline__ unsigned long long ld_acquire_u64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

// Grid-wide barrier of the NT consumer threads (threads 0 .. NT-1, named
// barrier 1) of every CTA. The arrival counter only grows: a launch's G CTAs
// take arrivals nG .. nG + G - 1 and each waits until the counter reaches
// (n + 1) G, so nothing is reset between barriers or launches. After a
// timeout the count is off a generation; moe_check_device, which reports the
// timeout, zeroes the header and with it the counter. One release per CTA (fence and
// add), one acquire load that sees the last arrival. False if it timed out.
// Writes before it are visible to ld.global.cg after it.
template <int NT>
__device__ bool grid_barrier(WsHeader* hdr, int site, int* s_flag, uint64_t limit, bool withhold) {
  auto consumer_sync = [] { asm volatile("bar.sync 1, %0;" ::"n"(NT) : "memory"); };
  consumer_sync();
  if (threadIdx.x == 0) {
    int ok = 1;
    unsigned long long* ctr = reinterpret_cast<unsigned long long*>(&hdr->bar_arrivals);
    const unsigned long long G = gridDim.x;
    __threadfence();
    // withhold (test aid): this CTA never arrives, so every other CTA's wait
    // runs out; the caller leaves as if it had timed out itself
    const unsigned long long arrival = withhold ? 0ull : atomicAdd(ctr, 1ull);
    const unsigned long long target = (arrival / G + 1) * G;
    if (withhold) {
      ok = 0;
    } else if (arrival + 1 < target) {
      const uint64_t t0 = globaltimer();
      while (ld_acquire_u64(ctr) < target) {
        if (globaltimer() - t0 > limit) {
          record_error(hdr, MOE_ERR_TIMEOUT, 100 + site);
          ok = 0;
          break;
        }
        __nanosleep(kBackoffNs);
      }
    } else {
      (void)ld_acquire_u64(ctr);  // the last arrival: acquire the others' writes
    }
    *s_flag = ok;
  }
  consumer_sync();
  return *s_flag != 0;
}

// Contributions to output rows a warp has stored but not yet counted (entry j
// of lane l: the counter index tok*H + row of a row that lane stored, or -1).
// Each output row y[t, n] counts its k + 1 contributions (k slot rows and the
// shared row) in DecodeArgs::sync after the kMaxSlots expert counters; the
// lane that brings the last one sums them in slot order and rounds once to
// bf16. A warp counts its list in one go (one fence for many rows).
template <int P>
struct Pending {
  int pend[P];
  int np;  // warp-uniform number of entries
};

// y[tok, row] = bf16(sum of the k slot rows in slot order + the shared row).
__device__ __forceinline__ void combine_row(const DecodeArgs& a, int idx) {
  const int tok = idx / a.H, row = idx - tok * a.H;
  float acc = 0.f;
  for (int j = 0; j < a.k; ++j) acc += __ldcg(a.y_slots + (int64_t)(tok * a.k + j) * a.H + row);
  if (a.ws_down != nullptr) acc += __ldcg(a.shared_out + (int64_t)tok * a.H + row);
  a.y[idx] = f32_to_bf16(acc);
}

// Count the pending contributions: one fence, then the counter increments;
// the lane that brings the last of an output row's k + 1 contributions
// combines it.
template <int P>
__device__ __forceinline__ void publish(const DecodeArgs& a, Pending<P>& q, int target) {
  __syncwarp();
  __threadfence();
  int32_t* rb_cnt = a.sync + kMaxSlots;
  int last = 0;
#pragma unroll
  for (int j = 0; j < P; ++j)
    if (j < q.np && q.pend[j] >= 0 && atomicAdd(rb_cnt + q.pend[j], 1) == target - 1) last |= 1 << j;
  if (last != 0) {
    __threadfence();
#pragma unroll
    for (int j = 0; j < P; ++j)
      if ((last >> j) & 1) combine_row(a, q.pend[j]);
  }
  q.np = 0;
}

template <int P>
__device__ __forceinline__ void add_pending(Pending<P>& q, int idx) {
#pragma unroll
  for (int j = 0; j < P; ++j)
    if (j == q.np) q.pend[j] = idx;
  ++q.np;
}

}  // namespace fused
}  // namespace moe
