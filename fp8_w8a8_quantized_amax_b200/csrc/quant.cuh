// quant.cuh -- bf16 -> E4M3 quantization kernels (HBM-bound).
//
// Every unit (a row, a 128-group of a row, a 128x128 block) is read once into
// registers with 16-byte loads, its amax found, and its codes written:
//   scale = amax / 448 (IEEE fp32 division; 1 when amax == 0)
//   code  = cvt.rn.satfinite.e4m3(x / scale)   (correctly rounded fp32 quotient first)
// The amax runs on the packed bf16 bit patterns: with the sign bit cleared,
// non-negative bf16 values order exactly like their 16-bit patterns, so an
// unsigned SIMD max over halfwords (__vmaxu2) is an exact max of |x|.
#pragma once

#include "ptx.cuh"

namespace fp8q {

// max(|a|, |b|) for each bf16 half (sign bit of the result is not meaningful).
__device__ __forceinline__ uint32_t absmax2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

__device__ __forceinline__ uint32_t absmax_bits_vec(const uint4& v, uint32_t acc) {
  return absmax2(absmax2(acc, v.x), absmax2(absmax2(v.y, v.z), v.w));
}

// Largest magnitude of the two halves as a 15-bit pattern.  Non-negative bf16
// values order exactly like their bit patterns, so an unsigned max is exact.
__device__ __forceinline__ uint32_t fold_halves(uint32_t m2) { return max(m2 & 0x7FFFu, (m2 >> 16) & 0x7FFFu); }

__device__ __forceinline__ float amax_bits_to_float(uint32_t bits16) { return __uint_as_float(bits16 << 16); }

__device__ __forceinline__ float scale_of(float amax) { return amax == 0.0f ? 1.0f : __fdiv_rn(amax, 448.0f); }

// The scale rounded to bf16 (the checkpoints' scale dtype) before the codes are
// computed; a scale that rounds to zero becomes 1 (all codes of its unit are 0).
__device__ __forceinline__ float scale_bf16(float s) {
  const float r = __bfloat162float(__float2bfloat16_rn(s));
  return r == 0.0f ? 1.0f : r;
}

// x / s, correctly rounded (identical to __fdiv_rn), for many x and one s.
// With y = RN(1/s) and q = RN(x * y) within one ulp of x / s, Markstein's
// correction step q' = RN(q + RN(x - q*s) * y) -- the residual x - q*s being
// exact in an FMA -- gives the correctly rounded quotient when nothing
// underflows or overflows (P. Markstein, "Computation of elementary functions
// on the IBM RISC System/6000 processor", IBM J. Res. Dev. 34(1), 1990).  Here
// |x / s| <= 448 * (1 + 2^-23); for s in [2^-60, 2^60] every intermediate of a
// quotient that can reach a nonzero E4M3 code stays normal, and quotients
// below 2^-11 encode to a signed zero either way.  Outside that range the
// plain IEEE division is used.  Three instructions per element instead of a
// division; the equality with __fdiv_rn is tested over every (amax, x) pair of
// bf16 values.
struct Divider {
  float s, y;
  bool fast;
};

__device__ __forceinline__ Divider make_divider(float s) {
  Divider d;
  d.s = s;
  d.fast = s >= 0x1p-60f && s <= 0x1p60f;
  d.y = __frcp_rn(s);
  return d;
}

// Codes of the two bf16 values packed in w (low half first), divided by s.
// The fast form runs on the negated values nx = -x (one xor of the two sign
// bits): q = nx * (-y) = x * y, r' = q * s - x = -r (exact in the FMA), and
// q' = q - r' * y = q + r * y: the same roundings as the textbook steps, and
// the signs come out right for x = +-0 as well (+0 + -0 would lose the sign
// of -0 in q + r * y; here the last FMA adds two zeros of x's sign).
// NEG: w holds the negated values already (a producer that can negate for
// free, such as the RMSNorm below, skips the xor).
template <bool FAST, bool NEG = false>
__device__ __forceinline__ uint32_t encode_pair(uint32_t w, const Divider& d, uint64_t ny2, uint64_t s2) {
  float ql, qh;
  if constexpr (FAST) {
    const uint32_t wn = NEG ? w : (w ^ 0x80008000u);
    const uint64_t nx2 = f32x2_pack(bf16lo(wn), bf16hi(wn));
    const uint64_t q2 = mul_f32x2(nx2, ny2);
    const uint64_t rn2 = fma_f32x2(q2, s2, nx2);
    f32x2_unpack(fma_f32x2(rn2, ny2, q2), ql, qh);
  } else {
    const uint32_t wp = NEG ? (w ^ 0x80008000u) : w;
    ql = __fdiv_rn(bf16lo(wp), d.s);
    qh = __fdiv_rn(bf16hi(wp), d.s);
  }
  return cvt_e4m3x2(ql, qh);
}

// 8 bf16 (one uint4) -> 8 codes (one uint2).
template <bool FAST, bool NEG = false>
__device__ __forceinline__ uint2 encode_vec(const uint4& v, const Divider& d) {
  const uint64_t ny2 = f32x2_pack(-d.y, -d.y);
  const uint64_t s2 = f32x2_pack(d.s, d.s);
  uint2 o;
  o.x = encode_pair<FAST, NEG>(v.x, d, ny2, s2) | (encode_pair<FAST, NEG>(v.y, d, ny2, s2) << 16);
  o.y = encode_pair<FAST, NEG>(v.z, d, ny2, s2) | (encode_pair<FAST, NEG>(v.w, d, ny2, s2) << 16);
  return o;
}

__device__ __forceinline__ uint4 ld_stream16(const void* p) {
  return __ldcs(reinterpret_cast<const uint4*>(p));
}

// ---------------------------------------------------------------- rows ---
// One CTA per row (per token of X, or per output channel of W).  Thread t
// holds vectors t, t + T, ..., t + (VPT-1) T of the row, T = blockDim.x.
template <int VPT>
__global__ void __launch_bounds__(1024) quant_rows_kernel(const uint16_t* __restrict__ x, int K, int64_t ldx,
                                                         uint8_t* __restrict__ q, int64_t ldq,
                                                         float* __restrict__ s, bool s16) {
  __shared__ uint32_t red[32];
  griddep_wait();
  griddep_launch_dependents();
  const int64_t r = blockIdx.x;
  const int nvec = K >> 3;
  const int T = blockDim.x;
  const uint16_t* xr = x + r * ldx;
  uint4 v[VPT];
  uint32_t m2 = 0;
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int idx = threadIdx.x + i * T;
    if (idx < nvec) {
      v[i] = ld_stream16(xr + idx * 8);
      m2 = absmax_bits_vec(v[i], m2);
    }
  }
  uint32_t m = __reduce_max_sync(0xFFFFFFFFu, fold_halves(m2));
  if (T > 32) {
    const int warp = threadIdx.x >> 5, nw = T >> 5;
    if (lane_id() == 0) red[warp] = m;
    __syncthreads();
    m = lane_id() < nw ? red[lane_id()] : 0u;
    m = __reduce_max_sync(0xFFFFFFFFu, m);
  }
  float sc = scale_of(amax_bits_to_float(m));
  if (s16) sc = scale_bf16(sc);
  if (threadIdx.x == 0) s[r] = sc;
  const Divider dv = make_divider(sc);
  uint8_t* qr = q + r * ldq;
  if (dv.fast) {
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      const int idx = threadIdx.x + i * T;
      if (idx < nvec) *reinterpret_cast<uint2*>(qr + idx * 8) = encode_vec<true>(v[i], dv);
    }
  } else {
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      const int idx = threadIdx.x + i * T;
      if (idx < nvec) *reinterpret_cast<uint2*>(qr + idx * 8) = encode_vec<false>(v[i], dv);
    }
  }
}

// ----------------------------------------------------- RMSNorm, then rows ---
// The input of the q/k/v and gate/up projections is RMSNorm(x) in bf16
// (Llama 3: RMSNorm before attention and MLP, eps 1e-5, kept in BF16).  One
// CTA per token normalises its row in registers and quantizes it per token,
// without writing the normalised bf16 row to memory:
//   ms = fl32(sum x^2 / K), rstd = rsqrt_rn(fl32(ms + eps)),
//   y = bf16(fl32(gamma * bf16(fl32(x * rstd)))), then y as quant_rows.
// The squares are exact in fp64 and summed in fp64 (in this kernel's order),
// so ms is the exact mean rounded once to fp32 unless that mean lies within a
// few fp64 roundings of an fp32 rounding boundary; rstd is written out when
// rstd != nullptr.

// -y for the 8 bf16 values of v (x) with the matching 8 of g (gamma), two at
// a time: -h = bf16(fl32(x * -rstd)) by a packed fp32 multiply and one bf16x2
// rounding; -y = bf16(gamma * -h) by one bf16x2 multiply.  The product of two
// bf16 values is exact in fp32, so rounding it once to bf16 (mul.rn.bf16x2)
// is the same as rounding the fp32 product.  Negation is exact and
// round-to-nearest-even is symmetric, so these are exactly the negated values
// of the textbook steps, as the encode wants them (encode_vec<..., true>);
// the amax ignores signs.
__device__ __forceinline__ uint32_t mul_bf16x2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}

__device__ __forceinline__ uint4 rmsnorm_vec(const uint4& v, const uint4& g, uint64_t rs2) {
  auto one = [&](uint32_t xw, uint32_t gw) -> uint32_t {
    float pl, ph;
    f32x2_unpack(mul_f32x2(f32x2_pack(bf16lo(xw), bf16hi(xw)), rs2), pl, ph);
    return mul_bf16x2(gw, pack_bf16x2(pl, ph));
  };
  return make_uint4(one(v.x, g.x), one(v.y, g.y), one(v.z, g.z), one(v.w, g.w));
}

// |x| of one bf16 value (its low 16 bits of b) as a double, by integer
// operations: the 15 magnitude bits move into the double's exponent and
// mantissa fields and the exponent is rebiased by 1023 - 127.  Exact for every
// normal bf16 value.  A zero or subnormal value becomes a double below 2^-126,
// whose square (under 2^-252) changes a row's sum of squares by less than
// 2^-236 in all: far below the sum's own fp64 rounding, and below fp32's
// smallest subnormal mean.
__device__ __forceinline__ double bf16_abs_f64(uint32_t b) {
  return __hiloint2double(static_cast<int>((b & 0x7FFFu) * 8192u + 0x38000000u), 0);
}
// The same for the high half of w, without a separate shift: (w & 0x7FFF0000) >> 3
// is the high word of the product with 2^29.
__device__ __forceinline__ double bf16hi_abs_f64(uint32_t w) {
  return __hiloint2double(static_cast<int>(__umulhi(w & 0x7FFF0000u, 0x20000000u) + 0x38000000u), 0);
}

// Squares of the 8 values of v (exact in fp64: 16 significant bits) added
// into four fp64 chains (one per 32-bit word), so that a thread's dependent
// fp64 additions per row are 2 * VPT long.
__device__ __forceinline__ void sumsq_vec(const uint4& v, double (&a)[4]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const double lo = bf16_abs_f64(w[i]), hi = bf16hi_abs_f64(w[i]);
    a[i] = fma(lo, lo, a[i]);
    a[i] = fma(hi, hi, a[i]);
  }
}

template <int VPT>
__global__ void __launch_bounds__(512) rmsnorm_quant_rows_kernel(const uint16_t* __restrict__ x,
                                                                 const uint16_t* __restrict__ gamma, int K,
                                                                 int64_t ldx, float eps, uint8_t* __restrict__ q,
                                                                 int64_t ldq, float* __restrict__ s,
                                                                 float* __restrict__ rstd) {
  __shared__ double red_sum[32];
  __shared__ uint32_t red_max[32];
  griddep_wait();
  griddep_launch_dependents();
  const int64_t r = blockIdx.x;
  const int nvec = K >> 3;
  const int T = blockDim.x;
  const int warp = threadIdx.x >> 5, nw = T >> 5;
  const uint16_t* xr = x + r * ldx;
  // gamma is read after the reductions (it is L1/L2-resident: every row reads
  // the same K values); holding it in registers from the start would cost a
  // third of the registers and so a third of the rows in flight per SM
  constexpr bool kGammaAhead = false;
  uint4 v[VPT], gv[kGammaAhead ? VPT : 1];
  double ssa[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int idx = threadIdx.x + i * T;
    if (idx < nvec) {
      v[i] = ld_stream16(xr + idx * 8);
      if constexpr (kGammaAhead) gv[i] = __ldg(reinterpret_cast<const uint4*>(gamma) + idx);
    }
  }
#pragma unroll
  for (int i = 0; i < VPT; ++i)
    if (threadIdx.x + i * T < nvec) sumsq_vec(v[i], ssa);
  double ss = (ssa[0] + ssa[1]) + (ssa[2] + ssa[3]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xFFFFFFFFu, ss, o);
  if (T > 32) {
    if (lane_id() == 0) red_sum[warp] = ss;
    __syncthreads();
    ss = lane_id() < nw ? red_sum[lane_id()] : 0.0;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xFFFFFFFFu, ss, o);
  }
  // mean of squares rounded once to fp32 (the double quotient first), then the
  // correctly rounded reciprocal square root of its IEEE sum with eps
  const float ms = __double2float_rn(ss / static_cast<double>(K));
  const float rs = __frsqrt_rn(__fadd_rn(ms, eps));
  if (threadIdx.x == 0 && rstd != nullptr) rstd[r] = rs;
  const uint64_t rs2 = f32x2_pack(-rs, -rs);   // v becomes -y (see rmsnorm_vec)
  uint32_t m2 = 0;
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    const int idx = threadIdx.x + i * T;
    if (idx < nvec) {
      if constexpr (kGammaAhead) v[i] = rmsnorm_vec(v[i], gv[i], rs2);
      else v[i] = rmsnorm_vec(v[i], __ldg(reinterpret_cast<const uint4*>(gamma) + idx), rs2);
      m2 = absmax_bits_vec(v[i], m2);
    }
  }
  uint32_t m = __reduce_max_sync(0xFFFFFFFFu, fold_halves(m2));
  if (T > 32) {
    if (lane_id() == 0) red_max[warp] = m;
    __syncthreads();
    m = lane_id() < nw ? red_max[lane_id()] : 0u;
    m = __reduce_max_sync(0xFFFFFFFFu, m);
  }
  const float sc = scale_of(amax_bits_to_float(m));
  if (threadIdx.x == 0) s[r] = sc;
  const Divider dv = make_divider(sc);
  uint8_t* qr = q + r * ldq;
  if (dv.fast) {
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      const int idx = threadIdx.x + i * T;
      if (idx < nvec) *reinterpret_cast<uint2*>(qr + idx * 8) = encode_vec<true, true>(v[i], dv);
    }
  } else {
#pragma unroll
    for (int i = 0; i < VPT; ++i) {
      const int idx = threadIdx.x + i * T;
      if (idx < nvec) *reinterpret_cast<uint2*>(qr + idx * 8) = encode_vec<false, true>(v[i], dv);
    }
  }
}

// --------------------------------------------------------- static scale ---
// Every element coded with one fixed, offline-calibrated scale (no amax),
// saturating beyond it; x_scale (when not null) is filled with that scale so
// that fp8_linear consumes the codes unchanged.  Grid-stride over the 16-byte
// vectors of all rows.
__global__ void __launch_bounds__(256) quant_static_kernel(const uint16_t* __restrict__ x, int64_t M, int K,
                                                          int64_t ldx, float sc, uint8_t* __restrict__ q,
                                                          int64_t ldq, float* __restrict__ s) {
  // 4 vectors per thread per round, all loads issued before any store, so
  // that 64 bytes per thread are in flight; vector u of a round is u * stride
  // further on (coalesced across the grid).  (row, vector) positions advance
  // incrementally in 32-bit arithmetic (the host keeps M * K / 8 below 2^31).
  constexpr int kVec = 4;
  griddep_wait();
  griddep_launch_dependents();
  const uint32_t nvec = static_cast<uint32_t>(K) >> 3;
  const uint32_t Mu = static_cast<uint32_t>(M);
  const uint32_t stride = gridDim.x * blockDim.x;
  const uint32_t st_m = stride / nvec, st_r = stride - st_m * nvec;
  const uint32_t i0 = blockIdx.x * blockDim.x + threadIdx.x;
  uint32_t m = i0 / nvec, r = i0 - m * nvec;
  auto advance = [&](uint32_t& mm, uint32_t& rr) {
    mm += st_m;
    rr += st_r;
    if (rr >= nvec) { rr -= nvec; ++mm; }
  };
  const Divider dv = make_divider(sc);
  while (m < Mu) {
    uint4 v[kVec];
    uint32_t mi[kVec], ri[kVec];
#pragma unroll
    for (int u = 0; u < kVec; ++u) {
      mi[u] = m;
      ri[u] = r;
      if (m < Mu) v[u] = ld_stream16(x + static_cast<int64_t>(m) * ldx + r * 8);
      advance(m, r);
    }
#pragma unroll
    for (int u = 0; u < kVec; ++u) {
      if (mi[u] < Mu) {
        *reinterpret_cast<uint2*>(q + static_cast<int64_t>(mi[u]) * ldq + ri[u] * 8) =
            dv.fast ? encode_vec<true>(v[u], dv) : encode_vec<false>(v[u], dv);
        if (s != nullptr && ri[u] == 0) s[mi[u]] = sc;
      }
    }
  }
}

// ----------------------------------------------------------- groups 128 ---
// Groups of 128 features: 16 consecutive lanes (a half warp) own one group,
// one 16-byte vector each.  Half warp h takes the groups h, h + H, h + 2H, ...
// of the row-major (token, group) list (H half warps in the grid), GPT of them
// in flight with all loads issued before any reduction.  The (token, group)
// position of each is advanced incrementally in 32-bit arithmetic: one
// division per half warp at the start, none in the loop.
template <int GPT>
__global__ void __launch_bounds__(256) quant_groups128_kernel(const uint16_t* __restrict__ x, int64_t M, int G,
                                                             int64_t ldx, uint8_t* __restrict__ q, int64_t ldq,
                                                             float* __restrict__ s, bool s16) {
  griddep_wait();
  griddep_launch_dependents();
  const int sub = threadIdx.x & 15;
  const uint32_t half_mask = 0xFFFFu << (threadIdx.x & 16);
  const uint32_t H = (gridDim.x * blockDim.x) >> 4;
  const uint32_t h = (blockIdx.x * blockDim.x + threadIdx.x) >> 4;
  const uint32_t Mu = static_cast<uint32_t>(M), Gu = static_cast<uint32_t>(G);
  const uint32_t step_m = H / Gu, step_g = H - step_m * Gu;   // (token, group) advance of H groups
  uint32_t m = h / Gu, g = h - m * Gu;                          // the half warp's next group
  auto advance = [&](uint32_t& mm, uint32_t& gg) {
    mm += step_m;
    gg += step_g;
    if (gg >= Gu) { gg -= Gu; ++mm; }
  };
  while (m < Mu) {
    uint4 v[GPT];
    uint32_t mi[GPT], gi[GPT];
    uint32_t mm = m, gg = g;
#pragma unroll
    for (int i = 0; i < GPT; ++i) {
      mi[i] = mm;
      gi[i] = gg;
      if (mm < Mu) v[i] = ld_stream16(x + static_cast<int64_t>(mm) * ldx + gg * 128 + sub * 8);
      advance(mm, gg);
    }
    m = mm;
    g = gg;
#pragma unroll
    for (int i = 0; i < GPT; ++i) {
      if (mi[i] < Mu) {  // uniform across the half warp
        // the half warp's max (each half warp reduces over its own 16 lanes)
        const uint32_t am = __reduce_max_sync(half_mask, fold_halves(absmax_bits_vec(v[i], 0u)));
        float sc = scale_of(amax_bits_to_float(am));
        if (s16) sc = scale_bf16(sc);
        if (sub == 0) s[static_cast<int64_t>(mi[i]) * Gu + gi[i]] = sc;
        const Divider dv = make_divider(sc);
        *reinterpret_cast<uint2*>(q + static_cast<int64_t>(mi[i]) * ldq + gi[i] * 128 + sub * 8) =
            dv.fast ? encode_vec<true>(v[i], dv) : encode_vec<false>(v[i], dv);
      }
    }
  }
}

// ---------------------------------------------------------- blocks 128 ---
// One CTA of 256 threads per 128 x 128 block of W.  Thread t owns the
// 16-byte vector (t % 16) of rows t/16 + 16 i, i < 8.  Rows past N are absent
// (the last row-block may be short) and take no part in the amax.
__global__ void __launch_bounds__(256) quant_blocks128_kernel(const uint16_t* __restrict__ w, int64_t N, int KB,
                                                             int64_t ldw, uint8_t* __restrict__ q, int64_t ldq,
                                                             float* __restrict__ s, bool s16) {
  __shared__ uint32_t red[8];
  griddep_wait();
  griddep_launch_dependents();
  const int kb = blockIdx.x;
  const int64_t nb = blockIdx.y;
  const int vc = threadIdx.x & 15;
  const int r0 = threadIdx.x >> 4;
  uint4 v[8];
  uint32_t m2 = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int64_t row = nb * 128 + r0 + 16 * i;
    if (row < N) {
      v[i] = ld_stream16(w + row * ldw + kb * 128 + vc * 8);
      m2 = absmax_bits_vec(v[i], m2);
    }
  }
  uint32_t m = __reduce_max_sync(0xFFFFFFFFu, fold_halves(m2));
  if (lane_id() == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  m = lane_id() < 8 ? red[lane_id()] : 0u;
  m = __reduce_max_sync(0xFFFFFFFFu, m);
  float sc = scale_of(amax_bits_to_float(m));
  if (s16) sc = scale_bf16(sc);
  if (threadIdx.x == 0) s[nb * KB + kb] = sc;
  const Divider dv = make_divider(sc);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int64_t row = nb * 128 + r0 + 16 * i;
    if (row < N)
      *reinterpret_cast<uint2*>(q + row * ldq + kb * 128 + vc * 8) =
          dv.fast ? encode_vec<true>(v[i], dv) : encode_vec<false>(v[i], dv);
  }
}

}  // namespace fp8q
