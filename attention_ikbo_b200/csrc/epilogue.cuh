// epilogue.cuh -- the per-group output epilogue of a ROCSified block, applied to one output
// row held in registers by one thread:
//     y = acc + bias[o]            GLM linear bias, section 3.1.2 Eq. (4), on the row axis
//     y = y + residual             pointwise merge of an aligned same-group input, section 3.1.3 Eq. (8)
//     y = Norm(y) * gamma + beta   group-local LayerNorm / RMSNorm over the row, section 3.1.3 Eq. (7)
//     y = act(y)                   pointwise activation, section 3.1.3 Eq. (8)
// ("ROCS: Request-Oriented Compute Sharing ...", arXiv:2607.27744).  The statistics of a row
// never leave the thread that owns it, so the norm needs no cross-thread reduction and reads
// only values of its own group.
#pragma once
#include "sm100.cuh"

namespace rocs {

enum { EPI_NORM_NONE = 0, EPI_NORM_LAYER = 1, EPI_NORM_RMS = 2 };
enum { EPI_ACT_NONE = 0, EPI_ACT_RELU = 1, EPI_ACT_SILU = 2, EPI_ACT_GELU = 3 };

struct EpiGroup {
  const float* bias;   // [o] or null
  const float* gamma;  // [row length] or null (1)
  const float* beta;   // [row length] or null (0)
  float eps;
  int norm;
  int act;
  int has_residual;
};

// Values travel in pairs (float2) so that adds and FMAs issue as the packed fp32x2 forms of
// sm_100 (__fadd2_rn / __ffma2_rn / __fmul2_rn): one instruction per two elements.
__device__ __forceinline__ float2 f2(float a) { return make_float2(a, a); }

// Row statistics accumulated one chunk at a time (the row is never held whole): LayerNorm merges
// each chunk's exact mean / sum of squared deviations into the running pair with the pairwise
// update of Chan, Golub and LeVeque (1979); RMSNorm sums squares.
struct RowStats {
  float n, mean, m2;
};

template <int N2>
__device__ __forceinline__ void stats_add_chunk(RowStats& s, const float2 (&x)[N2], int norm) {
  constexpr int N = 2 * N2;
  if (norm == EPI_NORM_LAYER) {
    float2 a[4] = {f2(0.0f), f2(0.0f), f2(0.0f), f2(0.0f)};
#pragma unroll
    for (int k = 0; k < N2; ++k) a[k & 3] = __fadd2_rn(a[k & 3], x[k]);
    const float2 a01 = __fadd2_rn(a[0], a[1]), a23 = __fadd2_rn(a[2], a[3]), at = __fadd2_rn(a01, a23);
    const float cm = (at.x + at.y) * (1.0f / N);
    const float2 ncm = f2(-cm);
    float2 q[4] = {f2(0.0f), f2(0.0f), f2(0.0f), f2(0.0f)};
#pragma unroll
    for (int k = 0; k < N2; ++k) {
      const float2 t = __fadd2_rn(x[k], ncm);
      q[k & 3] = __ffma2_rn(t, t, q[k & 3]);
    }
    const float2 q01 = __fadd2_rn(q[0], q[1]), q23 = __fadd2_rn(q[2], q[3]), qt = __fadd2_rn(q01, q23);
    const float cm2 = qt.x + qt.y;
    const float n = s.n + (float)N, delta = cm - s.mean;
    s.mean = fmaf(delta, (float)N / n, s.mean);
    s.m2 = s.m2 + cm2 + delta * delta * (s.n * (float)N / n);
    s.n = n;
  } else {
    float2 q[4] = {f2(0.0f), f2(0.0f), f2(0.0f), f2(0.0f)};
#pragma unroll
    for (int k = 0; k < N2; ++k) q[k & 3] = __ffma2_rn(x[k], x[k], q[k & 3]);
    const float2 q01 = __fadd2_rn(q[0], q[1]), q23 = __fadd2_rn(q[2], q[3]), qt = __fadd2_rn(q01, q23);
    s.m2 += qt.x + qt.y;
    s.n += (float)N;
  }
}

// mean (0 for RMSNorm) and 1/sqrt(var + eps) of a row of `len` values
__device__ __forceinline__ void stats_finish(const RowStats& s, int len, const EpiGroup& e, float& mean, float& inv) {
  mean = e.norm == EPI_NORM_LAYER ? s.mean : 0.0f;
  inv = rsqrtf(s.m2 / (float)len + e.eps);
}

// norm of one chunk: x = ((x - mean) * inv) * gamma + beta, gamma/beta at columns col0.. of the
// group's vectors in global memory (16-byte aligned, warp-uniform reads; null = 1 / 0)
template <int N2>
__device__ __forceinline__ void norm_chunk(float2 (&x)[N2], int col0, float mean, float inv, const EpiGroup& e) {
  const float2 inv2 = f2(inv), nm2 = f2(-mean * inv);
#pragma unroll
  for (int k2 = 0; k2 < N2 / 2; ++k2) {
    const float4 g = e.gamma ? __ldg(reinterpret_cast<const float4*>(e.gamma + col0) + k2) : make_float4(1.f, 1.f, 1.f, 1.f);
    const float4 b = e.beta ? __ldg(reinterpret_cast<const float4*>(e.beta + col0) + k2) : make_float4(0.f, 0.f, 0.f, 0.f);
    x[2 * k2] = __ffma2_rn(__ffma2_rn(x[2 * k2], inv2, nm2), make_float2(g.x, g.y), make_float2(b.x, b.y));
    x[2 * k2 + 1] = __ffma2_rn(__ffma2_rn(x[2 * k2 + 1], inv2, nm2), make_float2(g.z, g.w), make_float2(b.z, b.w));
  }
}

// the same with gamma/beta staged in shared memory (never null there)
template <int N2>
__device__ __forceinline__ void norm_chunk_smem(float2 (&x)[N2], const float* g, const float* b, float mean, float inv) {
  const float2 inv2 = f2(inv), nm2 = f2(-mean * inv);
#pragma unroll
  for (int k = 0; k < N2; ++k) {
    const float2 gv = reinterpret_cast<const float2*>(g)[k];
    const float2 bv = reinterpret_cast<const float2*>(b)[k];
    x[k] = __ffma2_rn(__ffma2_rn(x[k], inv2, nm2), gv, bv);
  }
}

__device__ __forceinline__ float tanh_approx(float x) {  // hardware tanh (max relative error about 2^-11)
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// GELU(x) = x/2 (1 + erf(x / sqrt 2)) with erf from Abramowitz & Stegun, Handbook of Mathematical
// Functions, formula 7.1.26 (|error| <= 1.5e-7): for z >= 0, erf z = 1 - P(t) exp(-z^2),
// t = 1 / (1 + p z), P(t) = a1 t + ... + a5 t^5.  With q = P(t) exp(-z^2), z = |x| / sqrt 2:
// 1 + erf(x / sqrt 2) = 2 - q for x >= 0 and q for x < 0.
__device__ __forceinline__ float gelu_as(float x) {
  const float z = fabsf(x) * 0.7071067811865476f;
  const float t = __fdividef(1.0f, fmaf(0.3275911f, z, 1.0f));
  float P = fmaf(1.061405429f, t, -1.453152027f);
  P = fmaf(P, t, 1.421413741f);
  P = fmaf(P, t, -0.284496736f);
  P = fmaf(P, t, 0.254829592f);
  P *= t;
  const float q = P * __expf(-z * z);
  return 0.5f * x * (x >= 0.0f ? 2.0f - q : q);
}

template <int ACT>
__device__ __forceinline__ float2 act_pair(float2 x) {
  if constexpr (ACT == EPI_ACT_RELU) return make_float2(fmaxf(x.x, 0.0f), fmaxf(x.y, 0.0f));
  // SiLU: x * sigmoid(x) with sigmoid(x) = (1 + tanh(x/2)) / 2, i.e. h + h * tanh(h) for h = x/2:
  // one MUFU operation per element
  if constexpr (ACT == EPI_ACT_SILU) {
    const float2 h = __fmul2_rn(x, f2(0.5f));
    return __ffma2_rn(h, make_float2(tanh_approx(h.x), tanh_approx(h.y)), h);
  }
  if constexpr (ACT == EPI_ACT_GELU) return make_float2(gelu_as(x.x), gelu_as(x.y));
  return x;
}

// activation fixed at compile time (the candidate group's, on the hot path)
template <int ACT, int N2>
__device__ __forceinline__ void act_chunk(float2 (&x)[N2]) {
  if constexpr (ACT != EPI_ACT_NONE) {
#pragma unroll
    for (int k = 0; k < N2; ++k) x[k] = act_pair<ACT>(x[k]);
  }
}

// activation chosen at run time, once per chunk (the request group's)
template <int N2>
__device__ __forceinline__ void act_chunk_rt(int act, float2 (&x)[N2]) {
  switch (act) {
    case EPI_ACT_RELU: act_chunk<EPI_ACT_RELU>(x); break;
    case EPI_ACT_SILU: act_chunk<EPI_ACT_SILU>(x); break;
    case EPI_ACT_GELU: act_chunk<EPI_ACT_GELU>(x); break;
    default: break;
  }
}

}  // namespace rocs
