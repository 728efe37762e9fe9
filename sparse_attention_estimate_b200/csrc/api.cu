// api.cu - the C ABI (include/vs.h): workspace layout, context, host-side
// argument validation, and the order in which each call enqueues its kernels.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <atomic>
#include <mutex>

#include "internal.cuh"

namespace vs {

static thread_local char g_msg[512] = "no error";

vs_status set_error(vs_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
  va_end(ap);
  return s;
}

vs_status cuda_check(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return VS_OK;
  return set_error(VS_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

static std::atomic<unsigned long long> g_launches{0};

vs_status launched(const char* what) {
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return cuda_check(cudaGetLastError(), what);
}

static size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

Layout make_layout(const vs_attn_cfg& cfg, int64_t max_seq, int64_t max_chunk) {
  Layout L{};
  const int64_t hq = cfg.hq, hkv = cfg.hkv, g = cfg.hq / cfg.hkv;
  L.e_pad = round_up(max_seq, kTile);
  L.rows_pad = round_up(max_chunk, 2 * kTile);
  L.nvar = cfg.dca_enabled ? 3 : 1;
  L.ntile = static_cast<int>(ceil_div(g * kEstRows, kTile));
  L.nsplit_max = 256;
  L.nwords = L.e_pad / 32 + kSPad + 8;
  L.npairs = L.rows_pad / (2 * kTile);
  L.nblk = L.e_pad / kTile;
  // DCA key chunks: the gather groups never straddle one, so each has one DCA class
  L.nkmax = cfg.dca_enabled ? ceil_div(max_seq, cfg.dca_chunk_size - cfg.dca_local_window) + 1 : 1;
  L.gcap = L.nblk + L.nkmax + 1;
  L.nsched = L.nblk + L.gcap;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = align_up(off + bytes, 256);
    return o;
  };
  L.err = take(64);
  L.stats = take(8 * sizeof(unsigned long long));
  L.theta = take(kHalf * sizeof(double));
  L.k_cont = take(static_cast<size_t>(hkv) * max_seq * kD * 2);
  L.k_dca = cfg.dca_enabled ? take(static_cast<size_t>(hkv) * max_seq * kD * 2) : 0;
  L.q_rot = take(static_cast<size_t>(L.nvar) * hq * L.rows_pad * kD * 2);
  L.q_est = take(static_cast<size_t>(hkv) * L.ntile * kTile * kD * 2);
  L.est_ml = take(static_cast<size_t>(L.nsplit_max) * hq * kEstRows * 2 * sizeof(float));
  L.lse_dca = take(static_cast<size_t>(hq) * kEstRows * sizeof(float));
  L.part_v = take(static_cast<size_t>(hq) * 2 * L.e_pad * sizeof(float));
  L.part_s = take(static_cast<size_t>(hq) * 4 * (L.e_pad + 256) * sizeof(float));
  L.thr = take(static_cast<size_t>(hq) * 2 * kMaxLevels * 2 * sizeof(uint32_t));
  L.lvl = take(static_cast<size_t>(hq) * 2 * L.e_pad);
  L.sel_state = take(sel_state_bytes(static_cast<int>(hq)));
  L.sel_part = take(sel_part_bytes(static_cast<int>(hq), kRecallLevels));
  L.hist = take(static_cast<size_t>(L.nsplit_max) * hq * kMaxLevels * sizeof(float));
  L.choice = take(static_cast<size_t>(hq) * 4 * sizeof(int32_t));
  L.base_rc = take(static_cast<size_t>(hq) * 2 * sizeof(int32_t));
  L.base_part = take(static_cast<size_t>(hq) * kBaseSplits * sizeof(double));
  L.vbits = take(static_cast<size_t>(hq) * L.nwords * sizeof(uint32_t));
  L.sbits = take(static_cast<size_t>(hq) * L.nwords * sizeof(uint32_t));
  L.scum = take(static_cast<size_t>(hq) * (L.nwords + 1) * sizeof(uint32_t));
  L.gbits = take(static_cast<size_t>(hq) * L.nwords * sizeof(uint32_t));
  L.gcum = take(static_cast<size_t>(hq) * (L.nwords + 1) * sizeof(uint32_t));
  L.gscan = take(static_cast<size_t>(hq) * (L.nblk + 1) * sizeof(int32_t));
  L.glist = take(static_cast<size_t>(hq) * L.e_pad * sizeof(int32_t));
  L.gtab = take(static_cast<size_t>(hq) * L.gcap * 4 * sizeof(int32_t));
  L.gkoff = take(static_cast<size_t>(hq) * (L.nkmax + 1) * sizeof(int32_t));
  L.sched = take(static_cast<size_t>(hq) * L.npairs * 2 * L.nsched * sizeof(int32_t));
  L.sched_cnt = take(static_cast<size_t>(hq) * L.npairs * sizeof(int32_t));
  L.sweep = take(static_cast<size_t>(hkv) * sizeof(int32_t));
  L.total = off;
  return L;
}

static PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

vs_status make_tmap_rows(CUtensorMap* map, const void* base, int64_t heads, int64_t rows,
                         int64_t head_stride_rows, int box_rows) {
  auto enc = get_encode_fn();
  if (!enc) return set_error(VS_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(kD), static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(heads)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(kD * 2),
                           static_cast<cuuint64_t>(head_stride_rows) * kD * 2};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                   box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return set_error(VS_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return VS_OK;
}

}  // namespace vs

using namespace vs;

// ------------------------------------------------------------------ validation helpers
static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static SelScratch sel_scratch(vs_ctx* c) {
  return SelScratch{ws_ptr<uint32_t>(c, c->L.thr), ws_ptr<uint8_t>(c, c->L.lvl), c->L.e_pad,
                    c->ws + c->L.sel_state, ws_ptr<uint32_t>(c, c->L.sel_part), c->err};
}

static vs_status check_cfg(const vs_attn_cfg* cfg) {
  VS_REQUIRE(cfg, VS_ERR_INVALID_ARG, "cfg is NULL");
  VS_REQUIRE(cfg->head_dim == kD, VS_ERR_UNSUPPORTED, "head_dim %d: only 128 is supported",
             cfg->head_dim);
  VS_REQUIRE(cfg->hq > 0 && cfg->hkv > 0, VS_ERR_INVALID_ARG, "head counts must be positive");
  VS_REQUIRE(cfg->hq % cfg->hkv == 0, VS_ERR_UNSUPPORTED, "hq (%d) must be a multiple of hkv (%d)",
             cfg->hq, cfg->hkv);
  VS_REQUIRE(cfg->hq / cfg->hkv <= kMaxG, VS_ERR_UNSUPPORTED, "GQA group %d > %d unsupported",
             cfg->hq / cfg->hkv, kMaxG);
  VS_REQUIRE(cfg->last_q >= 1 && cfg->last_q <= kEstRows, VS_ERR_INVALID_ARG,
             "last_q must be in [1, 64]");
  VS_REQUIRE(std::isfinite(cfg->softmax_scale) && cfg->softmax_scale > 0, VS_ERR_INVALID_ARG,
             "softmax_scale must be positive and finite");
  VS_REQUIRE(std::isfinite(cfg->rope_base) && cfg->rope_base > 1.0, VS_ERR_INVALID_ARG,
             "rope_base must be > 1");
  if (cfg->dca_enabled) {
    VS_REQUIRE(cfg->dca_chunk_size > 0 && cfg->dca_local_window >= 0 &&
                   cfg->dca_local_window < cfg->dca_chunk_size,
               VS_ERR_INVALID_ARG, "DCA needs 0 <= W < C");
    VS_REQUIRE(cfg->dca_chunk_size % kTile == 0 && cfg->dca_local_window % kTile == 0,
               VS_ERR_UNSUPPORTED, "DCA chunk size and local window must be multiples of 128");
  }
  return VS_OK;
}

static vs_status check_ctx(vs_ctx* c) {
  VS_REQUIRE(c, VS_ERR_INVALID_ARG, "context is NULL");
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_check(e, "cudaGetDevice");
  VS_REQUIRE(dev == c->device, VS_ERR_INVALID_ARG, "current device %d differs from the context's %d",
             dev, c->device);
  return VS_OK;
}

static vs_status check_tensor(const void* p, const char* name) {
  VS_REQUIRE(p, VS_ERR_INVALID_ARG, "%s is NULL", name);
  VS_REQUIRE(aligned16(p), VS_ERR_INVALID_ARG, "%s is not 16-byte aligned", name);
  return VS_OK;
}


// ------------------------------------------------------------------ context
extern "C" vs_status vs_workspace_size(const vs_attn_cfg* cfg, int64_t max_seq, int64_t max_chunk,
                                       size_t* bytes) {
  VS_TRY(check_cfg(cfg));
  VS_REQUIRE(bytes, VS_ERR_INVALID_ARG, "bytes is NULL");
  VS_REQUIRE(max_seq >= 1 && max_seq <= (int64_t(1) << 30), VS_ERR_INVALID_ARG,
             "max_seq out of range");
  VS_REQUIRE(max_chunk >= 1 && max_chunk <= max_seq, VS_ERR_INVALID_ARG,
             "max_chunk must be in [1, max_seq]");
  *bytes = make_layout(*cfg, max_seq, max_chunk).total;
  return VS_OK;
}

extern "C" vs_status vs_context_create(const vs_attn_cfg* cfg, int64_t max_seq, int64_t max_chunk,
                                       void* workspace, size_t ws_bytes, cudaStream_t stream,
                                       vs_ctx** out) {
  size_t need = 0;
  VS_TRY(vs_workspace_size(cfg, max_seq, max_chunk, &need));
  VS_REQUIRE(out, VS_ERR_INVALID_ARG, "out is NULL");
  VS_REQUIRE(workspace, VS_ERR_WORKSPACE, "workspace is NULL");
  VS_REQUIRE((reinterpret_cast<uintptr_t>(workspace) & 255u) == 0, VS_ERR_WORKSPACE,
             "workspace must be 256-byte aligned");
  VS_REQUIRE(ws_bytes >= need, VS_ERR_WORKSPACE, "workspace has %zu bytes, %zu needed", ws_bytes,
             need);
  int dev = 0;
  VS_TRY(cuda_check(cudaGetDevice(&dev), "cudaGetDevice"));
  int major = 0, minor = 0, sms = 0;
  VS_TRY(cuda_check(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev),
                    "cudaDeviceGetAttribute"));
  VS_TRY(cuda_check(cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev),
                    "cudaDeviceGetAttribute"));
  VS_TRY(cuda_check(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev),
                    "cudaDeviceGetAttribute"));
  VS_REQUIRE(major == 10 && minor == 0, VS_ERR_UNSUPPORTED,
             "device %d is sm_%d%d; this library is built for sm_100a (B200)", dev, major, minor);
  vs_ctx* c = static_cast<vs_ctx*>(calloc(1, sizeof(vs_ctx)));
  VS_REQUIRE(c, VS_ERR_INVALID_ARG, "host allocation failed");
  c->cfg = *cfg;
  c->max_seq = max_seq;
  c->max_chunk = max_chunk;
  c->ws = static_cast<char*>(workspace);
  c->ws_bytes = ws_bytes;
  c->L = make_layout(*cfg, max_seq, max_chunk);
  c->device = dev;
  c->num_sms = sms;
  c->wait_ns = 2000000000ull;
  c->deterministic = false;
  c->dca.enabled = cfg->dca_enabled ? 1 : 0;
  c->dca.C = cfg->dca_chunk_size;
  c->dca.W = cfg->dca_local_window;
  c->dca.S = cfg->dca_chunk_size - cfg->dca_local_window;
  c->err = ws_ptr<int>(c, c->L.err);
  c->stats = ws_ptr<unsigned long long>(c, c->L.stats);
  c->theta = ws_ptr<double>(c, c->L.theta);
  // theta_m = 1 / base^(2m/d) in fp64 (host libm pow)
  double th[kHalf];
  for (int m = 0; m < kHalf; ++m) th[m] = 1.0 / std::pow(cfg->rope_base, (2.0 * m) / kD);
  vs_status s = cuda_check(cudaMemsetAsync(c->ws, 0, c->L.k_cont, stream), "workspace init");
  if (s == VS_OK)
    s = cuda_check(cudaMemsetAsync(c->ws + c->L.q_est, 0, c->L.est_ml - c->L.q_est, stream),
                   "workspace init");
  if (s == VS_OK)
    s = cuda_check(
        cudaMemcpyAsync(c->theta, th, sizeof(th), cudaMemcpyHostToDevice, stream), "theta upload");
  // the host array must outlive the copy
  if (s == VS_OK) s = cuda_check(cudaStreamSynchronize(stream), "context init sync");
  if (s != VS_OK) {
    free(c);
    return s;
  }
  *out = c;
  return VS_OK;
}

extern "C" vs_status vs_context_destroy(vs_ctx* c) {
  free(c);
  return VS_OK;
}

extern "C" vs_status vs_context_reset(vs_ctx* c) {
  VS_REQUIRE(c, VS_ERR_INVALID_ARG, "context is NULL");
  c->kc = KCache{};
  c->kd = KCache{};
  return VS_OK;
}

extern "C" vs_status vs_set_wait_limit(vs_ctx* c, uint64_t ns) {
  VS_REQUIRE(c, VS_ERR_INVALID_ARG, "context is NULL");
  VS_REQUIRE(ns >= 1000, VS_ERR_INVALID_ARG, "wait limit below 1 us");
  c->wait_ns = ns;
  return VS_OK;
}

extern "C" vs_status vs_set_deterministic(vs_ctx* c, int on) {
  VS_REQUIRE(c, VS_ERR_INVALID_ARG, "context is NULL");
  c->deterministic = on != 0;
  return VS_OK;
}

extern "C" const char* vs_last_error(void) { return g_msg; }

// ------------------------------------------------------------------ calls
extern "C" vs_status dca_remap(vs_ctx* c, int64_t pos0, int64_t n, int32_t* pk, int32_t* pq_intra,
                               int32_t* pq_succ, int32_t* pq_inter, cudaStream_t st) {
  VS_TRY(check_ctx(c));
  VS_REQUIRE(pos0 >= 0 && n >= 0 && pos0 + n <= (int64_t(1) << 31), VS_ERR_INVALID_ARG,
             "positions out of int32 range");
  VS_REQUIRE(n == 0 || pk || pq_intra || pq_succ || pq_inter, VS_ERR_INVALID_ARG,
             "no output table given");
  return launch_dca_remap(c, pos0, n, pk, pq_intra, pq_succ, pq_inter, st);
}

static vs_status rotate_estimation_rows(vs_ctx* c, const uint16_t* q, int64_t q_rows,
                                        int64_t q_pos0, int64_t e, int* nr_out) {
  (void)q_rows;
  const int64_t r0 = std::max(q_pos0, e - static_cast<int64_t>(c->cfg.last_q));
  *nr_out = static_cast<int>(e - r0);
  return VS_OK;
}

static vs_status check_est_args(vs_ctx* c, const uint16_t* q, int64_t q_rows, int64_t q_pos0,
                                const uint16_t* k, int64_t k_rows, int64_t e) {
  VS_TRY(check_tensor(q, "q"));
  VS_TRY(check_tensor(k, "k"));
  VS_REQUIRE(e >= 1 && e <= c->max_seq, VS_ERR_UNSUPPORTED, "e=%lld outside [1, max_seq=%lld]",
             (long long)e, (long long)c->max_seq);
  VS_REQUIRE(e <= k_rows, VS_ERR_INVALID_ARG, "e exceeds k_rows");
  VS_REQUIRE(q_pos0 >= 0 && q_pos0 < e && e <= q_pos0 + q_rows, VS_ERR_INVALID_ARG,
             "q rows [q_pos0, q_pos0+q_rows) must contain the estimation rows ending at e");
  return VS_OK;
}

static vs_status prepare_estimation(vs_ctx* c, const uint16_t* q, int64_t q_rows, int64_t q_pos0,
                                    const uint16_t* k, int64_t k_rows, int64_t e, cudaStream_t st,
                                    int* nr) {
  VS_TRY(ensure_keys_rotated(c, k, k_rows, e, false, st));
  VS_TRY(rotate_estimation_rows(c, q, q_rows, q_pos0, e, nr));
  const int g = c->cfg.hq / c->cfg.hkv;
  return launch_rope_rows(c, reinterpret_cast<const bf16*>(q), q_rows, e - *nr - q_pos0,
                          ws_ptr<bf16>(c, c->L.q_est), 0, 0, g,
                          static_cast<int64_t>(c->L.ntile) * kTile, kEstRows, *nr, c->cfg.hq,
                          e - *nr, 0, st);
}

extern "C" vs_status vs_estimate(vs_ctx* c, const uint16_t* q, int64_t q_rows, int64_t q_pos0,
                                 const uint16_t* k, int64_t k_rows, int64_t e, float* vert,
                                 float* slash, int64_t e_ld, float* lse, cudaStream_t st) {
  VS_TRY(check_ctx(c));
  VS_TRY(check_est_args(c, q, q_rows, q_pos0, k, k_rows, e));
  VS_TRY(check_tensor(vert, "vert"));
  VS_TRY(check_tensor(slash, "slash"));
  VS_TRY(check_tensor(lse, "lse"));
  VS_REQUIRE(e_ld >= e, VS_ERR_INVALID_ARG, "e_ld < e");
  int nr = 0;
  VS_TRY(prepare_estimation(c, q, q_rows, q_pos0, k, k_rows, e, st, &nr));
  return run_estimate(c, q, q_rows, q_pos0, k, k_rows, e, vert, slash, e_ld, lse, st);
}

static vs_status check_sets(const int32_t* v_idx, int32_t cap_v, const int32_t* v_cnt,
                            const int32_t* s_off, int32_t cap_s, const int32_t* s_cnt) {
  VS_REQUIRE(v_idx && v_cnt && s_off && s_cnt, VS_ERR_INVALID_ARG, "set pointers must not be NULL");
  VS_REQUIRE(cap_v >= 1 && cap_s >= 1, VS_ERR_INVALID_ARG, "caps must be positive");
  return VS_OK;
}

extern "C" vs_status vs_select(vs_ctx* c, const float* vert, const float* slash, int64_t e_ld,
                               int64_t e, const int32_t* kv_budget, const int32_t* ks_budget,
                               int32_t* v_idx, int32_t cap_v, int32_t* v_cnt, int32_t* s_off,
                               int32_t cap_s, int32_t* s_cnt, cudaStream_t st) {
  VS_TRY(check_ctx(c));
  VS_TRY(check_tensor(vert, "vert"));
  VS_TRY(check_tensor(slash, "slash"));
  VS_REQUIRE(kv_budget && ks_budget, VS_ERR_INVALID_ARG, "budgets are NULL");
  VS_REQUIRE(e >= 1 && e <= c->max_seq && e_ld >= e, VS_ERR_INVALID_ARG, "bad e / e_ld");
  VS_TRY(check_sets(v_idx, cap_v, v_cnt, s_off, cap_s, s_cnt));
  return launch_select(sel_scratch(c), c->cfg.hq, vert, slash, e_ld, e, kv_budget, ks_budget, 1, nullptr,
                       v_idx, cap_v, v_cnt, s_off, cap_s, s_cnt, true, true, st);
}

extern "C" vs_status vs_refine(vs_ctx* c, const uint16_t* q, int64_t q_rows, int64_t q_pos0,
                               const uint16_t* k, int64_t k_rows, int64_t e, const float* vert,
                               const float* slash, int64_t e_ld, const float* lse, float tau,
                               int32_t max_iters, int32_t* kv_budget, int32_t* ks_budget,
                               int32_t* v_idx, int32_t cap_v, int32_t* v_cnt, int32_t* s_off,
                               int32_t cap_s, int32_t* s_cnt, float* recall, cudaStream_t st) {
  VS_TRY(check_ctx(c));
  VS_TRY(check_est_args(c, q, q_rows, q_pos0, k, k_rows, e));
  VS_TRY(check_tensor(vert, "vert"));
  VS_TRY(check_tensor(slash, "slash"));
  VS_TRY(check_tensor(lse, "lse"));
  VS_REQUIRE(e_ld >= e, VS_ERR_INVALID_ARG, "e_ld < e");
  VS_REQUIRE(kv_budget && ks_budget && recall, VS_ERR_INVALID_ARG, "budgets/recall are NULL");
  VS_REQUIRE(std::isfinite(tau), VS_ERR_INVALID_ARG, "tau must be finite");
  VS_REQUIRE(max_iters >= 0, VS_ERR_INVALID_ARG, "max_iters must be >= 0");
  VS_TRY(check_sets(v_idx, cap_v, v_cnt, s_off, cap_s, s_cnt));
  // levels t = 0..nlev-1 with budgets min(base * 2^t, e); beyond log2(e) + 1 doublings
  // every budget is saturated
  int sat = 1;
  while ((int64_t(1) << (sat - 1)) < e && sat < kMaxLevels) ++sat;
  const int nlev = std::min(std::min(max_iters, kRecallLevels - 1) + 1, sat + 1);
  int nr = 0;
  VS_TRY(prepare_estimation(c, q, q_rows, q_pos0, k, k_rows, e, st, &nr));
  VS_TRY(launch_select(sel_scratch(c), c->cfg.hq, vert, slash, e_ld, e, kv_budget, ks_budget, nlev, nullptr,
                       v_idx, cap_v, v_cnt, s_off, cap_s, s_cnt, true, false, st));
  const bool dca_recall = c->cfg.refine_dca_positions && c->dca.enabled;
  if (dca_recall) {
    VS_TRY(run_recall_hist_dca(c, q, q_rows, q_pos0, k, k_rows, e, nr, nlev, st));
  } else {
    // heads whose base budgets already reach tau need no histogram of the higher levels
    VS_TRY(run_recall_base(c, vert, slash, e_ld, e, nr, lse, tau, st));
    VS_TRY(run_recall_hist(c, e, nr, lse, nlev, st, ws_ptr<int>(c, c->L.base_rc) + c->cfg.hq));
  }
  VS_TRY(run_refine_decide(c, e, nr, nlev, tau, kv_budget, ks_budget, recall, !dca_recall, st));
  return launch_select(sel_scratch(c), c->cfg.hq, vert, slash, e_ld, e, kv_budget, ks_budget, nlev,
                       ws_ptr<int32_t>(c, c->L.choice), v_idx, cap_v, v_cnt, s_off, cap_s, s_cnt, false, true,
                       st);
}

extern "C" vs_status vs_calibrate_accumulate(vs_ctx* c, const int32_t* kv_budget, const int32_t* ks_budget,
                                             int32_t* kv_acc, int32_t* ks_acc, cudaStream_t st) {
  VS_TRY(check_ctx(c));
  VS_REQUIRE(kv_budget && ks_budget && kv_acc && ks_acc, VS_ERR_INVALID_ARG, "budget pointers must not be NULL");
  return run_budgets_max(c->cfg.hq, kv_budget, ks_budget, kv_acc, ks_acc, st);
}

extern "C" vs_status vs_sparse_prefill(vs_ctx* c, const uint16_t* q, int64_t q_rows,
                                       int64_t q_pos0, int64_t e, const uint16_t* k,
                                       const uint16_t* v, int64_t kv_rows, const int32_t* v_idx,
                                       int32_t cap_v, const int32_t* v_cnt, const int32_t* s_off,
                                       int32_t cap_s, const int32_t* s_cnt, uint16_t* out,
                                       float* lse_out, cudaStream_t st) {
  VS_TRY(check_ctx(c));
  VS_TRY(check_tensor(q, "q"));
  VS_TRY(check_tensor(k, "k"));
  VS_TRY(check_tensor(v, "v"));
  VS_TRY(check_tensor(out, "out"));
  VS_REQUIRE(!lse_out || aligned16(lse_out), VS_ERR_INVALID_ARG, "lse_out is not 16-byte aligned");
  VS_TRY(check_sets(v_idx, cap_v, v_cnt, s_off, cap_s, s_cnt));
  VS_REQUIRE(q_pos0 >= 0 && q_pos0 % kTile == 0, VS_ERR_UNSUPPORTED,
             "q_pos0 must be a multiple of 128");
  VS_REQUIRE(e > q_pos0 && e - q_pos0 <= q_rows, VS_ERR_INVALID_ARG,
             "rows [q_pos0, e) must lie in q");
  VS_REQUIRE(e - q_pos0 <= c->max_chunk, VS_ERR_UNSUPPORTED, "chunk of %lld rows > max_chunk",
             (long long)(e - q_pos0));
  VS_REQUIRE(e <= kv_rows && e <= c->max_seq, VS_ERR_INVALID_ARG, "e exceeds kv_rows or max_seq");
  return run_sparse_prefill(c, q, q_rows, q_pos0, e, k, v, kv_rows, v_idx, cap_v, v_cnt, s_off,
                            cap_s, s_cnt, out, lse_out, st);
}

extern "C" vs_status vs_prefill_stats(vs_ctx* c, cudaStream_t st, int64_t* out2) {
  VS_TRY(check_ctx(c));
  VS_REQUIRE(out2, VS_ERR_INVALID_ARG, "out2 is NULL");
  unsigned long long h[2] = {0, 0};
  VS_TRY(cuda_check(cudaMemcpyAsync(h, c->stats, sizeof(h), cudaMemcpyDeviceToHost, st),
                    "stats readback"));
  VS_TRY(cuda_check(cudaStreamSynchronize(st), "stats sync"));
  out2[0] = static_cast<int64_t>(h[0]);
  out2[1] = static_cast<int64_t>(h[1]);
  return VS_OK;
}

extern "C" vs_status vs_set_prefill_events(vs_ctx* c, cudaEvent_t start, cudaEvent_t stop) {
  VS_REQUIRE(c, VS_ERR_INVALID_ARG, "context is NULL");
  VS_REQUIRE((start == nullptr) == (stop == nullptr), VS_ERR_INVALID_ARG,
             "give both events or neither");
  c->ev_start = start;
  c->ev_stop = stop;
  return VS_OK;
}

extern "C" uint64_t vs_kernel_launches(void) { return g_launches.load(); }

extern "C" vs_status vs_status_poll(vs_ctx* c, cudaStream_t st) {
  VS_TRY(check_ctx(c));
  int h = 0;
  VS_TRY(cuda_check(cudaMemcpyAsync(&h, c->err, sizeof(int), cudaMemcpyDeviceToHost, st),
                    "error word readback"));
  VS_TRY(cuda_check(cudaStreamSynchronize(st), "status sync"));
  if (h != 0) {
    VS_TRY(cuda_check(cudaMemsetAsync(c->err, 0, 3 * sizeof(int), st), "error word clear"));
    VS_TRY(cuda_check(cudaStreamSynchronize(st), "status sync"));
    if (h == kDevErrTimeout)
      return set_error(VS_ERR_TIMEOUT, "a bounded device wait ran out");
    if (h == 5)
      return set_error(VS_ERR_DEVICE_CHECK,
                       "the keys changed under a cached rotation (call vs_context_reset after rewriting K)");
    return set_error(VS_ERR_DEVICE_CHECK, "device check failed (code %d)", h);
  }
  return VS_OK;
}

extern "C" vs_status vs_selftest_wait_timeout(vs_ctx* c, uint64_t limit_ns, cudaStream_t st) {
  VS_TRY(check_ctx(c));
  VS_REQUIRE(limit_ns >= 1000 && limit_ns <= 10000000000ull, VS_ERR_INVALID_ARG,
             "limit must be in [1 us, 10 s]");
  return launch_wait_selftest(c, limit_ns, st);
}
