// rope.cu - rotary position embedding of query/key rows at continuous or DCA
// positions, the rotated-key caches of a context, and dca_remap.
//
// RoPE follows the rotary code of the long-context essay (deepseekmodel.com,
// section 2.4): inverse frequency theta_m = 1/base^(2m/d), rotate-half pairs
// (m, m + d/2): y[m] = x[m] cos - x[m+64] sin, y[m+64] = x[m+64] cos + x[m] sin.
// The angle p * theta_m, its cosine and sine, and the products are evaluated in
// fp64 with every operation rounded separately (no fused multiply-add), then the
// result is rounded once to bf16 (nearest, ties to even): the operand the tensor
// cores consume. DCA positions follow the Qwen2.5-1M explainer, "Length
// Extrapolation" (intra-, successive- and inter-chunk patterns).
#include "internal.cuh"

namespace vs {

// Round a double to the nearest bf16 (ties to even). Dropping the low 45 of the
// 52 fraction bits with round-to-nearest-even leaves a value with 8 significant
// bits, exactly representable in fp32, whose upper 16 bits are the bf16 code.
__device__ __forceinline__ uint16_t f64_to_bf16_rne(double x) {
  unsigned long long b = static_cast<unsigned long long>(__double_as_longlong(x));
  const unsigned long long lsb = (b >> 45) & 1ull;
  b = (b + ((1ull << 44) - 1ull) + lsb) & ~((1ull << 45) - 1ull);
  const float f = static_cast<float>(__longlong_as_double(static_cast<long long>(b)));
  return static_cast<uint16_t>(__float_as_uint(f) >> 16);
}

__device__ __forceinline__ double bf16_bits_to_f64(uint16_t u) {
  return static_cast<double>(__uint_as_float(static_cast<uint32_t>(u) << 16));
}

// One thread per (row, 8 consecutive rotary pairs): 16-byte loads and stores of
// x[m0..m0+7] and x[m0+64..m0+71]; 32 rows per 256-thread block. Each thread
// evaluates its 8 cos/sin pairs once and applies them to every head.
constexpr int kRopePairs = 8;
__global__ void __launch_bounds__(256) rope_rows_kernel(
    const uint16_t* __restrict__ in, int64_t in_rows, int64_t in_row0, uint16_t* __restrict__ out,
    int64_t out_row0, int gdiv, int64_t gstride, int64_t hstride, int64_t nrows, int nheads,
    int64_t pos0, int mode, DcaParams dca, const double* __restrict__ theta) {
  const int64_t r = static_cast<int64_t>(blockIdx.x) * 32 + (threadIdx.x >> 3);
  const int m0 = (threadIdx.x & 7) * kRopePairs;
  if (r >= nrows) return;
  const int64_t t = pos0 + r;
  int64_t p;
  if (mode == 0)
    p = t;
  else if (mode == 1)
    p = dca_key_pos(t, dca);
  else
    p = dca_query_pos(t, mode - 2, dca);
  double s[kRopePairs], c[kRopePairs];
#pragma unroll
  for (int q = 0; q < kRopePairs; ++q) sincos(__dmul_rn(static_cast<double>(p), theta[m0 + q]), &s[q], &c[q]);
  for (int h = 0; h < nheads; ++h) {
    const uint16_t* x = in + (static_cast<int64_t>(h) * in_rows + in_row0 + r) * kD;
    const uint4 a = *reinterpret_cast<const uint4*>(x + m0);
    const uint4 b = *reinterpret_cast<const uint4*>(x + m0 + kHalf);
    const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w};
    uint32_t ya[4], yb[4];
#pragma unroll
    for (int q2 = 0; q2 < 4; ++q2) {
      uint32_t lo_a = 0, lo_b = 0;
#pragma unroll
      for (int k2 = 0; k2 < 2; ++k2) {
        const int q = 2 * q2 + k2;
        const double x1 = bf16_bits_to_f64(static_cast<uint16_t>(wa[q2] >> (16 * k2)));
        const double x2 = bf16_bits_to_f64(static_cast<uint16_t>(wb[q2] >> (16 * k2)));
        const uint32_t y1 = f64_to_bf16_rne(__dsub_rn(__dmul_rn(x1, c[q]), __dmul_rn(x2, s[q])));
        const uint32_t y2 = f64_to_bf16_rne(__dadd_rn(__dmul_rn(x2, c[q]), __dmul_rn(x1, s[q])));
        lo_a |= y1 << (16 * k2);
        lo_b |= y2 << (16 * k2);
      }
      ya[q2] = lo_a;
      yb[q2] = lo_b;
    }
    const int64_t orow = static_cast<int64_t>(h / gdiv) * gstride +
                         static_cast<int64_t>(h % gdiv) * hstride + out_row0 + r;
    uint16_t* y = out + orow * kD;
    *reinterpret_cast<uint4*>(y + m0) = make_uint4(ya[0], ya[1], ya[2], ya[3]);
    *reinterpret_cast<uint4*>(y + m0 + kHalf) = make_uint4(yb[0], yb[1], yb[2], yb[3]);
  }
}

vs_status launch_rope_rows(vs_ctx* c, const bf16* in, int64_t in_rows, int64_t in_row0, bf16* out,
                           int64_t out_rows, int64_t out_row0, int out_gdiv, int64_t out_gstride,
                           int64_t out_hstride, int64_t nrows, int nheads, int64_t pos0, int mode,
                           cudaStream_t st) {
  (void)out_rows;
  if (nrows <= 0) return VS_OK;
  const int64_t blocks = ceil_div(nrows, 32);
  rope_rows_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(
      reinterpret_cast<const uint16_t*>(in), in_rows, in_row0, reinterpret_cast<uint16_t*>(out),
      out_row0, out_gdiv, out_gstride, out_hstride, nrows, nheads, pos0, mode, c->dca, c->theta);
  return launched("rope_rows_kernel launch");
}

// Guard of a reused rotated-key cache: re-rotates kKCheckRows rows spread over [0, valid)
// of every KV head and compares them bit for bit with the cache; a difference (the
// caller rewrote K under the same pointer without vs_context_reset) raises the device
// error word. One block per sampled row, one thread per (head, rotary pair).
constexpr int kKCheckRows = 8;
constexpr int kDevErrKCache = 5;
__global__ void kcache_check_kernel(const uint16_t* __restrict__ k, int64_t k_rows, const uint16_t* __restrict__ cache,
                                    int64_t cache_rows, int64_t valid, int nheads, int mode, DcaParams dca,
                                    const double* __restrict__ theta, int* err) {
  const int64_t r = valid <= 1 ? 0 : (valid - 1) * blockIdx.x / (kKCheckRows - 1);
  const int64_t p = mode == 1 ? dca_key_pos(r, dca) : r;
  for (int w = threadIdx.x; w < nheads * kHalf; w += blockDim.x) {
    const int h = w / kHalf, m = w % kHalf;
    const uint16_t* x = k + (static_cast<int64_t>(h) * k_rows + r) * kD;
    const uint16_t* y = cache + (static_cast<int64_t>(h) * cache_rows + r) * kD;
    double sn, cs;
    sincos(__dmul_rn(static_cast<double>(p), theta[m]), &sn, &cs);
    const double x1 = bf16_bits_to_f64(x[m]), x2 = bf16_bits_to_f64(x[m + kHalf]);
    const uint16_t y1 = f64_to_bf16_rne(__dsub_rn(__dmul_rn(x1, cs), __dmul_rn(x2, sn)));
    const uint16_t y2 = f64_to_bf16_rne(__dadd_rn(__dmul_rn(x2, cs), __dmul_rn(x1, sn)));
    if (y1 != y[m] || y2 != y[m + kHalf]) atomicCAS(err, 0, kDevErrKCache);
  }
}

// Extends a rotated-key cache to rows [0, e). The cache is keyed on the source
// pointer and its row count; rows already rotated are assumed unchanged, which a
// sampled re-rotation checks on the device whenever the cache is reused.
vs_status ensure_keys_rotated(vs_ctx* c, const uint16_t* k, int64_t k_rows, int64_t e, bool dca,
                              cudaStream_t st) {
  KCache& kc = dca ? c->kd : c->kc;
  if (kc.src != k || kc.src_rows != k_rows) {
    kc.src = k;
    kc.src_rows = k_rows;
    kc.valid = 0;
  }
  if (kc.valid > 0) {
    kcache_check_kernel<<<kKCheckRows, 256, 0, st>>>(k, k_rows,
                                                    reinterpret_cast<const uint16_t*>(c->ws + (dca ? c->L.k_dca : c->L.k_cont)),
                                                    c->max_seq, kc.valid, c->cfg.hkv, dca ? 1 : 0, c->dca, c->theta,
                                                    c->err);
    vs_status s = launched("kcache_check_kernel launch");
    if (s != VS_OK) return s;
  }
  if (e <= kc.valid) return VS_OK;
  bf16* dst = ws_ptr<bf16>(c, dca ? c->L.k_dca : c->L.k_cont);
  const int64_t r0 = kc.valid;
  vs_status s = launch_rope_rows(c, reinterpret_cast<const bf16*>(k), k_rows, r0, dst, c->max_seq,
                                 r0, 1, c->max_seq, 0, e - r0, c->cfg.hkv, r0, dca ? 1 : 0, st);
  if (s != VS_OK) return s;
  kc.valid = e;
  return VS_OK;
}

__global__ void dca_remap_kernel(int64_t pos0, int64_t n, DcaParams dca, int32_t* pk, int32_t* pqi,
                                 int32_t* pqs, int32_t* pqx) {
  const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const int64_t t = pos0 + i;
  if (pk) pk[i] = static_cast<int32_t>(dca_key_pos(t, dca));
  if (pqi) pqi[i] = static_cast<int32_t>(dca_query_pos(t, 0, dca));
  if (pqs) pqs[i] = static_cast<int32_t>(dca_query_pos(t, 1, dca));
  if (pqx) pqx[i] = static_cast<int32_t>(dca_query_pos(t, 2, dca));
}

vs_status launch_dca_remap(vs_ctx* c, int64_t pos0, int64_t n, int32_t* pk, int32_t* pqi,
                           int32_t* pqs, int32_t* pqx, cudaStream_t st) {
  if (n == 0) return VS_OK;
  dca_remap_kernel<<<static_cast<unsigned>(ceil_div(n, 256)), 256, 0, st>>>(pos0, n, c->dca, pk,
                                                                           pqi, pqs, pqx);
  return launched("dca_remap_kernel launch");
}

}  // namespace vs
