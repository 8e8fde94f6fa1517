// calib.cuh -- static-scale calibration: the lo / hi quantiles of a bf16
// calibration tensor, exactly, from a histogram of its bit patterns.
//
// "Llama 3 精读实录" section 2 (FP8 量化实操) calibrates a static scale from
// percentiles of a calibration set (its 0.1% and 99.9% quantiles as the
// range, instead of min / max).  Reading: amax = max(|q(lo)|, |q(hi)|) with
// q(p) the linear interpolation between the order statistics at ranks
// floor(p (n - 1)) and the next one, in double; scale = fl32(fl32(amax) / 448),
// or 1 when amax is 0.
//
// A bf16 value has 65536 bit patterns, so counting patterns gives every order
// statistic exactly.  Patterns are counted under a 16-bit key that orders
// like the values: a negative pattern b maps to ~b, a non-negative one to
// b | 0x8000 (-0 and +0 get neighbouring keys; both are the value 0).
#pragma once

#include "ptx.cuh"

namespace fp8q {
namespace calib {

constexpr int kBins = 65536;

__device__ __forceinline__ uint32_t order_key(uint32_t b) {
  return (b & 0x8000u) ? (~b & 0xFFFFu) : (b | 0x8000u);
}

__device__ __forceinline__ double key_value(uint32_t key) {
  const uint32_t b = (key & 0x8000u) ? (key & 0x7FFFu) : (~key & 0xFFFFu);
  return static_cast<double>(__uint_as_float(b << 16));
}

// Count every element's key: 16-byte loads, grid-stride over the rows' vectors.
__global__ void __launch_bounds__(256) hist_kernel(const uint16_t* __restrict__ x, int64_t M, int K, int64_t ldx,
                                                   uint32_t* __restrict__ hist) {
  griddep_wait();
  griddep_launch_dependents();
  const int nvec = K >> 3;
  const int64_t total = M * nvec;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += stride) {
    const int64_t m = i / nvec;
    const int vi = static_cast<int>(i - m * nvec);
    const uint4 v = __ldcs(reinterpret_cast<const uint4*>(x + m * ldx + vi * 8));
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      atomicAdd(hist + order_key(w[h] & 0xFFFFu), 1u);
      atomicAdd(hist + order_key(w[h] >> 16), 1u);
    }
  }
}

// One block of 1024 threads: thread t owns bins [64 t, 64 t + 64).  Finds the
// keys at the four ranks, interpolates the two quantiles in double (explicit
// round-to-nearest operations: no fused multiply-add), writes the scale and
// zeroes the histogram for the next call.
__global__ void __launch_bounds__(1024) select_kernel(uint32_t* __restrict__ hist, int64_t n, double lo, double hi,
                                                      float* __restrict__ scale) {
  __shared__ unsigned long long warp_sums[32];
  __shared__ uint32_t found[4];
  griddep_wait();
  griddep_launch_dependents();
  const int t = threadIdx.x;
  const int lane = t & 31, warp = t >> 5;
  unsigned long long local = 0;
  for (int i = 0; i < 64; ++i) local += hist[t * 64 + i];
  // exclusive prefix of the per-thread sums: within the warp, then across warps
  unsigned long long incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned long long v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  unsigned long long before = 0;
  for (int w = 0; w < warp; ++w) before += warp_sums[w];
  const unsigned long long start = before + incl - local;
  // ranks of the two order statistics of each quantile
  const double pos_lo = __dmul_rn(lo, static_cast<double>(n - 1));
  const double pos_hi = __dmul_rn(hi, static_cast<double>(n - 1));
  const int64_t i_lo = static_cast<int64_t>(floor(pos_lo)), i_hi = static_cast<int64_t>(floor(pos_hi));
  const int64_t rank[4] = {i_lo, i_lo + 1 < n ? i_lo + 1 : n - 1, i_hi, i_hi + 1 < n ? i_hi + 1 : n - 1};
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const unsigned long long want = static_cast<unsigned long long>(rank[r]);
    if (want >= start && want < start + local) {
      unsigned long long acc = start;
      for (int i = 0; i < 64; ++i) {
        acc += hist[t * 64 + i];
        if (want < acc) {
          found[r] = static_cast<uint32_t>(t * 64 + i);
          break;
        }
      }
    }
  }
  __syncthreads();   // every rank found (and every count read) before the bins are cleared
  if (t == 0) {
    auto interp = [](double a, double b, double pos, int64_t i) {
      return __dadd_rn(a, __dmul_rn(__dsub_rn(b, a), __dsub_rn(pos, static_cast<double>(i))));
    };
    const double q_lo = interp(key_value(found[0]), key_value(found[1]), pos_lo, i_lo);
    const double q_hi = interp(key_value(found[2]), key_value(found[3]), pos_hi, i_hi);
    const double amax = fmax(fabs(q_lo), fabs(q_hi));
    *scale = amax == 0.0 ? 1.0f : __fdiv_rn(__double2float_rn(amax), 448.0f);
  }
#pragma unroll
  for (int i = 0; i < 64; ++i) hist[t * 64 + i] = 0u;
}

}  // namespace calib
}  // namespace fp8q
