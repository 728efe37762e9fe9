// internal.cuh - definitions shared by the library's translation units: the
// context, the workspace layout, kernel parameter blocks and launch helpers.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/vs.h"
#include "sm100.cuh"

namespace vs {

using bf16 = __nv_bfloat16;

constexpr int kD = 128;          // head_dim
constexpr int kHalf = 64;        // rotary pairs
constexpr int kTile = 128;       // query rows per MMA tile / keys per key block
constexpr int kMaxG = 8;         // largest GQA group the estimation kernel tiles
constexpr int kMaxLevels = 32;   // selection levels stored per (head, array)
constexpr int kRecallLevels = 20;  // refinement levels (max_iters <= 19)
constexpr int kSPad = 4;         // zero words in front of each slash bitmap
constexpr int kBaseSplits = 32;  // CTAs per head of the base-recall scan
constexpr int kEstRows = 64;     // estimation rows per head (upper bound of last_q)

// Parameters every kernel with a bounded wait receives.
struct DevCommon {
  int* err;          // device error word
  uint64_t wait_ns;  // limit of each bounded wait
};

// DCA constants on the device (S = C - W).
struct DcaParams {
  int enabled;
  int64_t C, W, S;
};

__host__ __device__ inline int64_t dca_key_pos(int64_t t, const DcaParams& d) {
  return d.enabled ? t % d.S : t;
}
// cls: 0 intra, 1 successive, 2 inter
__host__ __device__ inline int64_t dca_query_pos(int64_t t, int cls, const DcaParams& d) {
  if (!d.enabled) return t;
  const int64_t r = t % d.S;
  if (cls == 0) return r;
  if (cls == 1) return (r + d.S < d.C - 1) ? r + d.S : d.C - 1;
  return d.C - 1;
}

// Workspace regions (byte offsets from the workspace base).
struct Layout {
  size_t err, stats, theta;
  size_t k_cont, k_dca;       // rotated key caches [hkv][max_seq][128]
  size_t q_rot;               // rotated chunk queries [nvar][hq][rows_pad][128]
  size_t q_est;               // rotated estimation rows [hkv][ntile*128][128]
  size_t est_ml;              // lse partials [nsplit_max][hq*64][2]
  size_t lse_dca;             // estimation rows' lse at DCA positions [hq][64]
  size_t part_v;              // vertical partial sums [hq][2][e_pad]
  size_t part_s;              // slash partial sums [hq][2 halves][2 lo/hi][e_pad + 128]
  size_t thr;                 // selection thresholds [hq][2][kMaxLevels] (key, take)
  size_t lvl;                 // levels [hq][2][max_seq] uint8
  size_t sel_state, sel_part; // radix-select state and per-segment histograms
  size_t hist;                // recall histograms [nsplit_max][hq][kMaxLevels]
  size_t choice;              // chosen level per head [hq] + flags
  size_t base_rc;             // recall at the base budgets [hq] fp32, then decided flags [hq] int
  size_t base_part;           // partial sums of the base-recall scan [hq][kBaseSplits] fp64
  size_t vbits, sbits, scum;  // bitmaps [hq][nwords] and slash prefix counts
  size_t gbits, gcum;         // gathered vertical columns [hq][nwords] and their prefix counts
  size_t gscan;               // gathered columns before each key block [hq][nblk + 1]
  size_t glist;               // gathered columns, ascending [hq][e_pad]
  size_t gtab;                // gather groups [hq][gcap] (start, count, DCA key chunk, first column)
  size_t gkoff;               // first group of each DCA key chunk [hq][nkmax + 1]
  size_t sched, sched_cnt;    // work lists [hq][npairs][2 * nsched] (each list written twice in a row)
                              // and their lengths [hq][npairs]
  size_t sweep;               // list position of each KV head's attention CTAs [hkv] (a hint)
  size_t total;
  int64_t rows_pad;           // max_chunk rounded up to 256
  int64_t e_pad;              // max_seq rounded up to 128
  int64_t nwords;             // bitmap words per head (incl. padding)
  int64_t npairs, nblk;       // query-tile pairs per chunk, key blocks per sequence
  int64_t nkmax;              // DCA key chunks a sequence can span (1 without DCA)
  int64_t gcap;               // gather groups per head, at most
  int64_t nsched;             // work-list entries per pair, at most (key blocks + groups)
  int nvar, ntile, nsplit_max;
};

Layout make_layout(const vs_attn_cfg& cfg, int64_t max_seq, int64_t max_chunk);

struct KCache {
  const void* src = nullptr;
  int64_t src_rows = 0;
  int64_t valid = 0;
};

}  // namespace vs

struct vs_ctx {
  vs_attn_cfg cfg;
  int64_t max_seq, max_chunk;
  char* ws;
  size_t ws_bytes;
  vs::Layout L;
  int device, num_sms;
  uint64_t wait_ns;
  bool deterministic;  // attention CTAs sweep their lists from the start
  vs::DcaParams dca;
  vs::KCache kc, kd;  // continuous / DCA rotated key caches
  int hist_nsplit;    // splits of the last recall-histogram launch
  cudaEvent_t ev_start, ev_stop;  // optional timing events around the attention kernel
  // device pointers into the workspace
  int* err;
  unsigned long long* stats;
  double* theta;
};

namespace vs {

template <class T>
inline T* ws_ptr(vs_ctx* c, size_t off) {
  return reinterpret_cast<T*>(c->ws + off);
}
inline DevCommon dev_common(vs_ctx* c) { return DevCommon{c->err, c->wait_ns}; }

// Error reporting (thread-local message).
vs_status set_error(vs_status s, const char* fmt, ...);

// Host-side checks: return the status (with the thread's error message set) from
// the enclosing function.
#define VS_REQUIRE(cond, code, ...)                   \
  do {                                                \
    if (!(cond)) return set_error(code, __VA_ARGS__); \
  } while (0)
#define VS_TRY(expr)            \
  do {                          \
    vs_status _s = (expr);      \
    if (_s != VS_OK) return _s; \
  } while (0)
vs_status cuda_check(cudaError_t e, const char* what);

// TMA descriptor for a [heads][rows][128] bf16 tensor: box of 64 columns x box_rows rows x 1 head,
// 128-byte swizzle. `rows` bounds the loads (rows beyond read as zero).
vs_status make_tmap_rows(CUtensorMap* map, const void* base, int64_t heads, int64_t rows,
                         int64_t head_stride_rows, int box_rows);

// ---------------------------------------------------------------- launchers (one per .cu file)
// rope.cu
vs_status launch_rope_rows(vs_ctx* c, const bf16* in, int64_t in_rows, int64_t in_row0, bf16* out,
                           int64_t out_rows, int64_t out_row0, int out_gdiv, int64_t out_gstride,
                           int64_t out_hstride, int64_t nrows, int nheads, int64_t pos0, int mode,
                           cudaStream_t st);
vs_status ensure_keys_rotated(vs_ctx* c, const uint16_t* k, int64_t k_rows, int64_t e, bool dca,
                              cudaStream_t st);
vs_status launch_dca_remap(vs_ctx* c, int64_t pos0, int64_t n, int32_t* pk, int32_t* pqi,
                           int32_t* pqs, int32_t* pqx, cudaStream_t st);
// estimate.cu
vs_status run_estimate(vs_ctx* c, const uint16_t* q, int64_t q_rows, int64_t q_pos0,
                       const uint16_t* k, int64_t k_rows, int64_t e, float* vert, float* slash,
                       int64_t e_ld, float* lse, cudaStream_t st);
vs_status run_recall_hist_dca(vs_ctx* c, const uint16_t* q, int64_t q_rows, int64_t q_pos0,
                              const uint16_t* k, int64_t k_rows, int64_t e, int nr, int nlev,
                              cudaStream_t st);
vs_status run_recall_hist(vs_ctx* c, int64_t e, int nr, const float* lse, int nlev,
                          cudaStream_t st, const int* dec = nullptr);
vs_status run_recall_base(vs_ctx* c, const float* vert, const float* slash, int64_t e_ld, int64_t e, int nr,
                          const float* lse, float tau, cudaStream_t st);
// select.cu
constexpr int kSelMaxSegments = 64;  // segments (CTAs) per (head, array), at most
// Scratch of the selection kernels (the context's workspace, or the no-alloc array).
struct SelScratch {
  uint32_t* thr;   // thresholds [hq][2][kMaxLevels][2] (key, how many equal keys to take)
  uint8_t* lvl;    // per-element levels [hq][2][e_pad]
  int64_t e_pad;
  void* state;     // radix-select state [hq][2] (sel_state_bytes)
  uint32_t* part;  // per-segment histograms and counts (sel_part_bytes)
  int* err;        // device error word
};
size_t sel_state_bytes(int hq);
size_t sel_part_bytes(int hq, int nslot);  // nslot: levels selected at once (1 for vs_select)
// Thresholds and levels of nlev budget levels (thresholds_and_levels), and/or the index
// lists of the chosen level per head (compact; choice nullptr: level 0).
vs_status launch_select(const SelScratch& sc, int hq, const float* vert, const float* slash, int64_t e_ld,
                        int64_t e, const int32_t* kv, const int32_t* ks, int nlev, const int32_t* choice,
                        int32_t* v_idx, int32_t cap_v, int32_t* v_cnt, int32_t* s_off, int32_t cap_s,
                        int32_t* s_cnt, bool thresholds_and_levels, bool compact, cudaStream_t st);
vs_status run_refine_decide(vs_ctx* c, int64_t e, int nr, int nlev, float tau, int32_t* kv,
                            int32_t* ks, float* recall, bool base_decided, cudaStream_t st);
vs_status run_budgets_max(int hq, const int32_t* kv, const int32_t* ks, int32_t* kv_acc, int32_t* ks_acc,
                          cudaStream_t st);
// attn.cu
vs_status run_sparse_prefill(vs_ctx* c, const uint16_t* q, int64_t q_rows, int64_t q_pos0,
                             int64_t e, const uint16_t* k, const uint16_t* v, int64_t kv_rows,
                             const int32_t* v_idx, int32_t cap_v, const int32_t* v_cnt,
                             const int32_t* s_off, int32_t cap_s, const int32_t* s_cnt,
                             uint16_t* out, float* lse_out, cudaStream_t st);
vs_status launch_wait_selftest(vs_ctx* c, uint64_t limit_ns, cudaStream_t st);

// Counts a kernel launch (vs_kernel_launches) and returns the launch error state.
vs_status launched(const char* what);

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline int64_t round_up(int64_t a, int64_t b) { return ceil_div(a, b) * b; }

}  // namespace vs
