// select.cu - top-k selection of vertical columns and slash offsets, and the
// refinement decision.
//
// The vertical-slash step of the Qwen2.5-1M explainer ("Sparse Attention",
// step 3) keeps, per head, the k_v columns with the largest vertical score and
// the k_s diagonal offsets with the largest slash score; "Sparsity Refinement"
// doubles both budgets while the head's attention recall is below the
// threshold. Every budget of a refinement run is a level t with
// k_t = min(k_base * 2^t, e); since the ranking (score descending, index
// ascending) is fixed, the selected sets are nested and one pass can assign each
// column / offset the first level that selects it.
//
// Kernels (one 1024-thread CTA per (head, array)):
//  thresholds_kernel  - radix select (four 8-bit digit passes over the fp32 bit
//                       pattern, which orders non-negative floats) of the k_t-th
//                       largest key for every level at once, plus how many
//                       elements equal to that key are taken (lowest index first)
//  levels_kernel      - ordered pass writing each element's first level (255: none)
//  compact_kernel     - ordered pass writing the ascending index list of a level
//  refine_decide_kernel - first level whose recall reaches tau (or saturation)
#include "internal.cuh"

namespace vs {

constexpr uint32_t kNoThreshold = 0xFFFFFFFFu;  // level with k = 0: selects nothing
constexpr int kDevErrCap = 3;                    // an output list was longer than its cap

// Sort key of element j: fp32 bit pattern of a non-negative score (0 for
// non-positive or NaN), +inf for slash offset 0, which is always selected.
__device__ __forceinline__ uint32_t sel_key(float x, int64_t j, int arr) {
  if (arr == 1 && j == 0) return 0x7F800000u;
  return (x > 0.0f) ? __float_as_uint(x) : 0u;
}

// Exclusive block-wide prefix sum of v (blockDim.x == 1024); *total gets the sum.
__device__ __forceinline__ int block_excl_scan(int v, int* wsum, int* total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) wsum[w] = x;
  __syncthreads();
  if (w == 0) {
    int s = wsum[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    wsum[lane] = s;
  }
  __syncthreads();
  const int base = (w > 0) ? wsum[w - 1] : 0;
  *total = wsum[31];
  __syncthreads();
  return base + x - v;
}

__global__ void __launch_bounds__(1024) thresholds_kernel(const float* __restrict__ vert,
                                                          const float* __restrict__ slash,
                                                          int64_t e_ld, int64_t e,
                                                          const int32_t* __restrict__ kv,
                                                          const int32_t* __restrict__ ks, int nlev,
                                                          uint32_t* __restrict__ thr) {
  const int h = blockIdx.x, arr = blockIdx.y, tid = threadIdx.x;
  const float* x = (arr == 0 ? vert : slash) + static_cast<int64_t>(h) * e_ld;
  __shared__ uint32_t hist[kMaxLevels][256];
  __shared__ uint32_t prefix[kMaxLevels], uprefix[kMaxLevels];
  __shared__ int64_t rank[kMaxLevels];
  __shared__ int slot_of[kMaxLevels], active[kMaxLevels];
  __shared__ int nuniq;
  if (tid < nlev) {
    int64_t base = (arr == 0) ? kv[h] : ks[h];
    if (base < 0) base = 0;
    int64_t k = base << tid;
    if (k > e || (tid > 0 && (base << (tid - 1)) >= e)) k = e;
    if (base == 0) k = 0;
    rank[tid] = k;
    prefix[tid] = 0;
    active[tid] = k > 0;
  }
  __syncthreads();
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    if (tid == 0) {
      int nu = 0;
      for (int t = 0; t < nlev; ++t) {
        slot_of[t] = -1;
        if (!active[t]) continue;
        int u = 0;
        while (u < nu && uprefix[u] != prefix[t]) ++u;
        if (u == nu) uprefix[nu++] = prefix[t];
        slot_of[t] = u;
      }
      nuniq = nu;
    }
    __syncthreads();
    const int nu = nuniq;
    for (int i = tid; i < nu * 256; i += blockDim.x) (&hist[0][0])[i] = 0;
    __syncthreads();
    for (int64_t j0 = 0; j0 < e; j0 += blockDim.x) {
      const int64_t j = j0 + tid;
      int u = -1;
      uint32_t digit = 0;
      if (j < e) {
        const uint32_t key = sel_key(x[j], j, arr);
        const uint32_t hp = (pass == 0) ? 0u : (key >> (shift + 8));
        for (int uu = 0; uu < nu; ++uu)
          if (uprefix[uu] == hp) {
            u = uu;
            break;
          }
        digit = (key >> shift) & 255u;
      }
      // aggregate equal (slot, digit) pairs of the warp into one atomic
      const uint32_t tag = (u < 0) ? 0xFFFFFFFFu : ((static_cast<uint32_t>(u) << 8) | digit);
      const uint32_t peers = __match_any_sync(0xffffffffu, tag);
      if (u >= 0 && (__ffs(peers) - 1) == (tid & 31))
        atomicAdd(&hist[u][digit], static_cast<uint32_t>(__popc(peers)));
    }
    __syncthreads();
    if (tid < nlev && active[tid]) {
      const int u = slot_of[tid];
      int64_t cum = 0;
      for (int d = 255; d >= 0; --d) {
        const int64_t cnt = hist[u][d];
        if (cum + cnt >= rank[tid]) {
          prefix[tid] = (prefix[tid] << 8) | static_cast<uint32_t>(d);
          rank[tid] -= cum;
          break;
        }
        cum += cnt;
      }
    }
    __syncthreads();
  }
  if (tid < kMaxLevels) {
    uint32_t* o = thr + ((static_cast<int64_t>(h) * 2 + arr) * kMaxLevels + tid) * 2;
    const bool ok = tid < nlev && active[tid];
    o[0] = ok ? prefix[tid] : kNoThreshold;
    o[1] = ok ? static_cast<uint32_t>(rank[tid]) : 0u;
  }
}

__global__ void __launch_bounds__(1024) levels_kernel(const float* __restrict__ vert,
                                                      const float* __restrict__ slash, int64_t e_ld,
                                                      int64_t e, int nlev,
                                                      const uint32_t* __restrict__ thr,
                                                      uint8_t* __restrict__ lvl, int64_t e_pad) {
  const int h = blockIdx.x, arr = blockIdx.y, tid = threadIdx.x;
  const float* x = (arr == 0 ? vert : slash) + static_cast<int64_t>(h) * e_ld;
  uint8_t* out = lvl + (static_cast<int64_t>(h) * 2 + arr) * e_pad;
  __shared__ uint32_t T[kMaxLevels], take[kMaxLevels], uT[kMaxLevels];
  __shared__ int64_t run[kMaxLevels];
  __shared__ int nu_s;
  __shared__ int wsum[32];
  if (tid == 0) {
    int nu = 0;
    for (int t = 0; t < nlev; ++t) {
      const uint32_t* p = thr + ((static_cast<int64_t>(h) * 2 + arr) * kMaxLevels + t) * 2;
      T[t] = p[0];
      take[t] = p[1];
      if (p[0] == kNoThreshold) continue;
      int u = 0;
      while (u < nu && uT[u] != p[0]) ++u;
      if (u == nu) {
        uT[nu] = p[0];
        run[nu] = 0;
        ++nu;
      }
    }
    nu_s = nu;
  }
  __syncthreads();
  const int nu = nu_s;
  for (int64_t j0 = 0; j0 < e; j0 += blockDim.x) {
    const int64_t j = j0 + tid;
    const bool valid = j < e;
    const uint32_t key = valid ? sel_key(x[j], j, arr) : 0u;
    int myu = -1;
    if (valid)
      for (int u = 0; u < nu; ++u)
        if (uT[u] == key) {
          myu = u;
          break;
        }
    int64_t myrank = 0;
    if (__syncthreads_or(myu >= 0)) {
      for (int u = 0; u < nu; ++u) {
        if (!__syncthreads_or(myu == u)) continue;
        int total = 0;
        const int r = block_excl_scan(myu == u ? 1 : 0, wsum, &total);
        if (myu == u) myrank = run[u] + r;
        __syncthreads();
        if (tid == 0) run[u] += total;
        __syncthreads();
      }
    }
    if (valid) {
      uint8_t level = 255;
      for (int t = 0; t < nlev; ++t) {
        const uint32_t tt = T[t];
        if (tt == kNoThreshold) continue;
        if (key > tt || (key == tt && myrank < static_cast<int64_t>(take[t]))) {
          level = static_cast<uint8_t>(t);
          break;
        }
      }
      out[j] = level;
    }
  }
}

__global__ void __launch_bounds__(1024) compact_kernel(const uint8_t* __restrict__ lvl,
                                                       int64_t e_pad, int64_t e,
                                                       const int32_t* __restrict__ choice,
                                                       int32_t* v_idx, int32_t cap_v,
                                                       int32_t* v_cnt, int32_t* s_off,
                                                       int32_t cap_s, int32_t* s_cnt, int* err) {
  const int h = blockIdx.x, arr = blockIdx.y, tid = threadIdx.x;
  const uint8_t* lv = lvl + (static_cast<int64_t>(h) * 2 + arr) * e_pad;
  const int tsel = choice ? choice[h] : 0;
  const int32_t cap = arr == 0 ? cap_v : cap_s;
  int32_t* out = arr == 0 ? v_idx + static_cast<int64_t>(h) * cap_v
                          : s_off + static_cast<int64_t>(h) * cap_s;
  __shared__ int wsum[32];
  int64_t running = 0;
  for (int64_t j0 = 0; j0 < e; j0 += blockDim.x) {
    const int64_t j = j0 + tid;
    const int flag = (j < e && static_cast<int>(lv[j]) <= tsel) ? 1 : 0;
    int total = 0;
    const int r = block_excl_scan(flag, wsum, &total);
    const int64_t pos = running + r;
    if (flag && pos < cap) out[pos] = static_cast<int32_t>(j);
    running += total;
  }
  if (tid == 0) {
    (arr == 0 ? v_cnt : s_cnt)[h] = static_cast<int32_t>(running < cap ? running : cap);
    if (running > cap) atomicCAS(err, 0, kDevErrCap);
  }
}

__global__ void refine_decide_kernel(const float* __restrict__ hist, int nsplit, int hq, int nlev,
                                     int nr, int64_t e, float tau, int32_t* kv, int32_t* ks,
                                     float* recall, int32_t* choice) {
  const int h = blockIdx.x * blockDim.x + threadIdx.x;
  if (h >= hq) return;
  int64_t kv0 = kv[h] < 0 ? 0 : kv[h], ks0 = ks[h] < 0 ? 0 : ks[h];
  double cum = 0.0;
  int chosen = nlev - 1;
  int64_t kvt = 0, kst = 0;
  double rc = 0.0;
  for (int t = 0; t < nlev; ++t) {
    double m = 0.0;
    for (int s = 0; s < nsplit; ++s)
      m += static_cast<double>(hist[(static_cast<int64_t>(s) * hq + h) * kMaxLevels + t]);
    cum = m;  // the histogram is cumulative: level t holds the recall mass of C_t
    rc = cum / nr;
    kvt = (kv0 << t) > e ? e : (kv0 << t);
    kst = (ks0 << t) > e ? e : (ks0 << t);
    if (t > 0 && (kv0 << (t - 1)) >= e) kvt = e;
    if (t > 0 && (ks0 << (t - 1)) >= e) kst = e;
    if (rc >= static_cast<double>(tau) || (kvt >= e && kst >= e) || t == nlev - 1) {
      chosen = t;
      break;
    }
  }
  choice[h] = chosen;
  kv[h] = static_cast<int32_t>(kvt);
  ks[h] = static_cast<int32_t>(kst);
  recall[h] = static_cast<float>(rc);
}

vs_status run_thresholds(vs_ctx* c, const float* vert, const float* slash, int64_t e_ld, int64_t e,
                         const int32_t* kv, const int32_t* ks, int nlev, cudaStream_t st) {
  thresholds_kernel<<<dim3(c->cfg.hq, 2), 1024, 0, st>>>(vert, slash, e_ld, e, kv, ks, nlev,
                                                        ws_ptr<uint32_t>(c, c->L.thr));
  return launched("thresholds_kernel launch");
}

vs_status run_levels(vs_ctx* c, const float* vert, const float* slash, int64_t e_ld, int64_t e,
                     int nlev, cudaStream_t st) {
  levels_kernel<<<dim3(c->cfg.hq, 2), 1024, 0, st>>>(vert, slash, e_ld, e, nlev,
                                                    ws_ptr<uint32_t>(c, c->L.thr),
                                                    ws_ptr<uint8_t>(c, c->L.lvl), c->L.e_pad);
  return launched("levels_kernel launch");
}

vs_status run_compact(vs_ctx* c, int64_t e, const int32_t* level_of_head, int32_t* v_idx,
                      int32_t cap_v, int32_t* v_cnt, int32_t* s_off, int32_t cap_s,
                      int32_t* s_cnt, cudaStream_t st) {
  compact_kernel<<<dim3(c->cfg.hq, 2), 1024, 0, st>>>(ws_ptr<uint8_t>(c, c->L.lvl), c->L.e_pad, e,
                                                     level_of_head, v_idx, cap_v, v_cnt, s_off,
                                                     cap_s, s_cnt, c->err);
  return launched("compact_kernel launch");
}

vs_status run_refine_decide(vs_ctx* c, int64_t e, int nr, int nlev, float tau, int32_t* kv,
                            int32_t* ks, float* recall, cudaStream_t st) {
  refine_decide_kernel<<<static_cast<unsigned>(ceil_div(c->cfg.hq, 64)), 64, 0, st>>>(
      ws_ptr<float>(c, c->L.hist), c->hist_nsplit, c->cfg.hq, nlev, nr, e, tau, kv, ks, recall,
      ws_ptr<int32_t>(c, c->L.choice));
  return launched("refine_decide_kernel launch");
}

// The three selection kernels on caller-given scratch pointers (no context):
// thr [hq][2][kMaxLevels][2] uint32, lvl [hq][2][e_pad] uint8, err one int.
vs_status launch_select_raw(int hq, const float* vert, const float* slash, int64_t e_ld, int64_t e,
                            const int32_t* kv, const int32_t* ks, uint32_t* thr, uint8_t* lvl,
                            int64_t e_pad, int* err, int32_t* v_idx, int32_t cap_v, int32_t* v_cnt,
                            int32_t* s_off, int32_t cap_s, int32_t* s_cnt, cudaStream_t st) {
  thresholds_kernel<<<dim3(hq, 2), 1024, 0, st>>>(vert, slash, e_ld, e, kv, ks, 1, thr);
  vs_status s = launched("thresholds_kernel launch");
  if (s != VS_OK) return s;
  levels_kernel<<<dim3(hq, 2), 1024, 0, st>>>(vert, slash, e_ld, e, 1, thr, lvl, e_pad);
  s = launched("levels_kernel launch");
  if (s != VS_OK) return s;
  compact_kernel<<<dim3(hq, 2), 1024, 0, st>>>(lvl, e_pad, e, nullptr, v_idx, cap_v, v_cnt, s_off,
                                              cap_s, s_cnt, err);
  return launched("compact_kernel launch");
}

}  // namespace vs
