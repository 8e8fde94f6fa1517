// gemv_w8a16.cuh -- weight-only FP8 linear for small M: bf16 activations
// times E4M3 weight codes dequantized in registers, fp32 sums, bf16 output.
//
// The layer that the "Llama-3.1-70B-FP8-Dynamic" explainer describes for GPUs
// without FP8 tensor cores (section 三, the GPU choice list; FAQ Q1): the
// checkpoint's weights stay FP8 in memory and are widened when the layer runs;
// the activations are not quantized.  For one token (and, on request, up to
// 16) the work is a weight stream (N * K code bytes against 2 * M * N * K
// flops), so it runs on the CUDA cores: a code is widened exactly (E4M3 -> f16
// -> f32; every E4M3 value is an f16 value), multiplied with the bf16
// activation widened to f32 and added in fp32 with packed f32x2 FMAs.  From two
// tokens on, the tensor-core variant of the decode kernel is faster (about 7
// CUDA-core instructions per code at eight tokens).
//
// A CTA owns R consecutive output channels and all of K.  One producer warp
// streams the R weight rows through a ring of shared-memory stages with bulk
// copies (kStageK codes of each row per stage), so that the bytes in flight
// per SM do not depend on the consumers' registers.  Eight consumer warps each
// take a fixed 512-code slice of every stage (16 codes per lane), read the
// matching activations (16 bf16 per token, through L1), and keep R x MT
// packed sums.  At the end each warp folds its lanes' sums with a
// transpose-reduce (lane l ends with the total of one (channel, token) pair),
// the warps' totals are added in shared memory in warp order, scaled by the
// channel's w_scale and written as bf16.
#pragma once

#include "ptx.cuh"

namespace fp8q {
namespace wonly {

constexpr int kConsumerWarps = 8;
constexpr int kThreads = 32 * (kConsumerWarps + 1);
constexpr int kLaneCodes = 16;                              // codes per lane per stage and row
constexpr int kStageK = kConsumerWarps * 32 * kLaneCodes;   // 4096 codes of each row per stage
constexpr int kMaxTokens = 16;

template <int R, int STAGES>
struct Layout {
  static constexpr int kStageBytes = R * kStageK;
  static constexpr int kBarOffset = STAGES * kStageBytes;
  static constexpr int kRedOffset = kBarOffset + 2 * STAGES * 8 + 16;   // full, empty, abort flag
  template <int V>
  static constexpr int bytes() {
    return kRedOffset + kConsumerWarps * V * 4;
  }
};

// Eight E4M3 codes -> eight fp32 values, packed in pairs (codes 2i, 2i+1).
__device__ __forceinline__ void widen8(uint32_t lo4, uint32_t hi4, uint64_t (&w)[4]) {
  const uint32_t v[2] = {lo4, hi4};
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    float f0, f1, f2, f3;
    asm("{\n\t.reg .b16 c01, c23, h0, h1, h2, h3;\n\t.reg .b32 p01, p23;\n\t"
        "mov.b32 {c01, c23}, %4;\n\t"
        "cvt.rn.f16x2.e4m3x2 p01, c01;\n\t"
        "cvt.rn.f16x2.e4m3x2 p23, c23;\n\t"
        "mov.b32 {h0, h1}, p01;\n\t"
        "mov.b32 {h2, h3}, p23;\n\t"
        "cvt.f32.f16 %0, h0;\n\t"
        "cvt.f32.f16 %1, h1;\n\t"
        "cvt.f32.f16 %2, h2;\n\t"
        "cvt.f32.f16 %3, h3;\n\t}"
        : "=f"(f0), "=f"(f1), "=f"(f2), "=f"(f3)
        : "r"(v[i]));
    w[2 * i] = f32x2_pack(f0, f1);
    w[2 * i + 1] = f32x2_pack(f2, f3);
  }
}

template <int V>
__host__ __device__ constexpr int log2_of() {
  return V <= 1 ? 0 : 1 + log2_of<V / 2>();
}

// Reduce V values (a power of two <= 32) across the warp's lanes.  Each of the
// log2(V) halving steps trades half of the values with the lane 16 >> s apart,
// so the vector shrinks as the lane groups do; the remaining steps are plain
// butterflies.  Lane l returns the total of value (l >> (5 - log2 V)).
template <int V>
__device__ __forceinline__ float transpose_reduce(float (&v)[V]) {
  constexpr int kLog = log2_of<V>();
  const uint32_t lane = lane_id();
#pragma unroll
  for (int s = 0; s < kLog; ++s) {
    const int h = V >> (s + 1);
    const int o = 16 >> s;
    const bool upper = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < h; ++i) {
      const float send = upper ? v[i] : v[i + h];
      const float keep = upper ? v[i + h] : v[i];
      v[i] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, o);
    }
  }
  float t = v[0];
#pragma unroll
  for (int s = kLog; s < 5; ++s) t += __shfl_xor_sync(0xFFFFFFFFu, t, 16 >> s);
  return t;
}

struct Params {
  const __nv_bfloat16* x;
  int64_t ldx;
  const uint8_t* w;
  const float* ws;
  __nv_bfloat16* y;
  int64_t ldy;
  int M, N, K;
};

// One bounded wait that ignores the abort flag: the teardown of a CTA whose
// copies may still be landing in its shared memory.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const uint32_t b = smem_u32(bar);
  const uint64_t t0 = globaltimer();
  while (!mbar_try_wait(b, parity)) {
    if (globaltimer() - t0 > kWaitLimitNs) {
      atomicCAS(&g_device_error, 0, static_cast<int>(kErrWaitDrain));
      return;
    }
  }
}

template <int MT, int R, int STAGES, int MINB>
__global__ void __launch_bounds__(kThreads, MINB) gemv_w8a16_kernel(const Params p) {
  using L = Layout<R, STAGES>;
  constexpr int V = R * MT;
  static_assert(V <= 32 && (V & (V - 1)) == 0, "R * MT must be a power of two <= 32");
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBarOffset);
  uint64_t* empty = full + STAGES;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + STAGES);
  float* red = reinterpret_cast<float*>(smem + L::kRedOffset);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * R;
  const int rows = min(R, p.N - n0);
  const int n_stages = (p.K + kStageK - 1) / kStageK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumerWarps);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  griddep_wait();

  if (warp == kConsumerWarps) {
    // ---- producer: R rows x up to kStageK codes per stage
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      int issued = 0;
      for (int i = 0; i < n_stages; ++i) {
        const int slot = i % STAGES;
        if (i >= STAGES && !mbar_wait(&empty[slot], ((i / STAGES) & 1) ^ 1u, abort_flag, kErrWaitEmpty)) break;
        const int k0 = i * kStageK;
        const uint32_t bytes = static_cast<uint32_t>(min(kStageK, p.K - k0));
        mbar_arrive_expect_tx(&full[slot], bytes * rows);
        uint8_t* dst = smem + slot * L::kStageBytes;
        for (int r = 0; r < rows; ++r)
          bulk_load(dst + r * kStageK, p.w + static_cast<int64_t>(n0 + r) * p.K + k0, bytes, &full[slot], pol);
        issued = i + 1;
      }
      // Copies of the last stages may still be landing if the consumers gave
      // up: wait for them before the CTA's shared memory goes away.
      if (*abort_flag) {
        for (int i = max(0, issued - STAGES); i < issued; ++i) drain_wait(&full[i % STAGES], (i / STAGES) & 1);
      }
    }
    griddep_launch_dependents();
    return;
  }

  // ---- consumers
  uint64_t acc[R][MT];
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int t = 0; t < MT; ++t) acc[r][t] = 0;

  const int col = warp * (32 * kLaneCodes) + lane * kLaneCodes;   // within a stage
  for (int i = 0; i < n_stages; ++i) {
    const int slot = i % STAGES;
    if (!__all_sync(0xFFFFFFFFu, mbar_wait(&full[slot], (i / STAGES) & 1, abort_flag, kErrWaitFull))) break;
    const int k = i * kStageK + col;
    if (k < p.K) {
      uint4 q[R];
      const uint8_t* st = smem + slot * L::kStageBytes + col;
#pragma unroll
      for (int r = 0; r < R; ++r) q[r] = *reinterpret_cast<const uint4*>(st + r * kStageK);
      // two halves of 8 codes: widened weights for one half of every row at a time
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint64_t w[R][4];
#pragma unroll
        for (int r = 0; r < R; ++r) widen8(h ? q[r].z : q[r].x, h ? q[r].w : q[r].y, w[r]);
#pragma unroll
        for (int t = 0; t < MT; ++t) {
          if (t < p.M) {
            const uint4 a = __ldg(reinterpret_cast<const uint4*>(p.x + t * p.ldx + k) + h);
            const uint32_t xv[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const uint64_t xf = f32x2_pack(bf16lo(xv[j]), bf16hi(xv[j]));
#pragma unroll
              for (int r = 0; r < R; ++r) acc[r][t] = fma_f32x2(xf, w[r][j], acc[r][t]);
            }
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[slot]);
  }

  float v[V];
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int t = 0; t < MT; ++t) {
      float lo, hi;
      f32x2_unpack(acc[r][t], lo, hi);
      v[r * MT + t] = lo + hi;
    }
  const float s = transpose_reduce<V>(v);
  constexpr int kShift = 5 - log2_of<V>();
  if ((lane & ((1 << kShift) - 1)) == 0) red[warp * V + (lane >> kShift)] = s;
  asm volatile("bar.sync 1, %0;" ::"n"(32 * kConsumerWarps) : "memory");
  if (threadIdx.x < V && !*abort_flag) {
    const int r = threadIdx.x / MT;
    const int t = threadIdx.x % MT;
    if (r < rows && t < p.M) {
      float sum = 0.f;
#pragma unroll
      for (int w8 = 0; w8 < kConsumerWarps; ++w8) sum += red[w8 * V + threadIdx.x];
      p.y[t * p.ldy + n0 + r] = __float2bfloat16_rn(sum * p.ws[n0 + r]);
    }
  }
}

}  // namespace wonly
}  // namespace fp8q
