// api.cu -- the exported C ABI of librswa.so (declared in include/rswa.h).
//
// Every entry point validates its arguments on the host before launching
// anything, records a message for rswa_last_error() on failure, and only
// enqueues work on the caller's stream.
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include <nvtx3/nvToolsExt.h>

#include "common.cuh"
#include "internal.h"

namespace {

// An NVTX range named after the entry point around each call that launches work (it shows
// in Nsight timelines; without an attached tool the calls are no-ops).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

thread_local char g_last_error[512] = "";

rswa_status fail(rswa_status code, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof g_last_error, fmt, ap);
  va_end(ap);
  return code;
}

rswa_status ok() {
  g_last_error[0] = '\0';
  return RSWA_OK;
}

rswa_status cuda_fail(cudaError_t e, const char* what) {
  return fail(RSWA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

#define REQUIRE_PTR(p)                                                                         \
  do {                                                                                         \
    if ((p) == nullptr) return fail(RSWA_ERR_INVALID, "%s: %s must not be NULL", fn, #p);     \
    if (!aligned16(p)) return fail(RSWA_ERR_INVALID, "%s: %s is not 16-byte aligned", fn, #p); \
  } while (0)

#define REQUIRE_PTR_OR_NULL(p)                                                                 \
  do {                                                                                         \
    if ((p) != nullptr && !aligned16(p))                                                       \
      return fail(RSWA_ERR_INVALID, "%s: %s is not 16-byte aligned", fn, #p);                  \
  } while (0)

rswa_status check_dims(const char* fn, const rswa_dims* d, bool need_prefix) {
  if (d == nullptr) return fail(RSWA_ERR_INVALID, "%s: dims must not be NULL", fn);
  if (d->batch < 1) return fail(RSWA_ERR_INVALID, "%s: batch must be >= 1 (got %d)", fn, d->batch);
  if (d->heads < 1 || d->heads > 128) return fail(RSWA_ERR_INVALID, "%s: heads must be in [1, 128] (got %d)", fn, d->heads);
  if (d->head_dim != rswa::kHeadDim)
    return fail(RSWA_ERR_UNSUPPORTED, "%s: head_dim must be 128 (got %d)", fn, d->head_dim);
  if (d->ring < 1 || d->ring > 1024) return fail(RSWA_ERR_INVALID, "%s: ring must be in [1, 1024] (got %d)", fn, d->ring);
  if (need_prefix && (d->prefix_cap < 0 || d->prefix_cap > (int64_t)1 << 30))
    return fail(RSWA_ERR_INVALID, "%s: prefix_cap out of range (got %lld)", fn, (long long)d->prefix_cap);
  if (d->batch > 65535) return fail(RSWA_ERR_UNSUPPORTED, "%s: batch above 65535", fn);
  return RSWA_OK;
}

int32_t* ws_status(void* ws) { return reinterpret_cast<int32_t*>(ws); }

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

// Set by rswa_test_arm_wait_timeout for the next decode launch of this host thread only.
thread_local int g_test_drop_tile = -1;
thread_local uint64_t g_test_wait_ns = 0;

}  // namespace

namespace rswa {
int device_sm_count() {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms > 0 ? sms : 148;
}
}  // namespace rswa

extern "C" {

const char* rswa_last_error(void) { return g_last_error; }

int32_t rswa_version(void) { return 5; }

size_t rswa_workspace_bytes(const rswa_dims* dims, int32_t op) {
  const char* fn = "rswa_workspace_bytes";
  if (check_dims(fn, dims, true) != RSWA_OK) return 0;
  switch (op) {
    case RSWA_OP_DECODE: {
      // sized for rswa_decode and for the fused rswa_decode_append (one tile more)
      const int64_t t = rswa::decode_max_tiles_dense(dims->prefix_cap, dims->ring);
      size_t most = 0;
      for (int64_t extra = 0; extra <= 1; ++extra) {
        const size_t b =
            rswa::plan_decode_workspace(dims->batch, dims->heads, t + extra, rswa::device_sm_count()).bytes;
        most = b > most ? b : most;
      }
      return most;
    }
    case RSWA_OP_SRSWA_DECODE: {
      // the plan depends on topk (and the fused append's extra tile): size for the largest
      size_t most = 0;
      for (int k = 1; k <= rswa::kMaxTopk; ++k)
        for (int64_t extra = 0; extra <= 1; ++extra) {
          const size_t b = rswa::plan_decode_workspace(dims->batch, dims->heads,
                                                       rswa::decode_max_tiles_sparse(k, dims->ring) + extra,
                                                       rswa::device_sm_count())
                               .bytes;
          most = b > most ? b : most;
        }
      return most;
    }
    case RSWA_OP_SRSWA_ROUTED: {
      // srswa_decode_routed / srswa_step: the SR-SWA decode plan (any topk, the step's extra
      // token tile) followed by the fused router's area
      size_t most = 0;
      for (int k = 1; k <= rswa::kMaxTopk; ++k)
        for (int64_t extra = 0; extra <= 1; ++extra) {
          const size_t b = rswa::plan_decode_workspace(dims->batch, dims->heads,
                                                       rswa::decode_max_tiles_sparse(k, dims->ring) + extra,
                                                       rswa::device_sm_count())
                               .bytes;
          most = b > most ? b : most;
        }
      return align256(most) + rswa::route_area_bytes(dims->batch, dims->prefix_cap);
    }
    case RSWA_OP_ROUTE:
    case RSWA_OP_PREFILL:
      return 256;
    default:
      fail(RSWA_ERR_INVALID, "%s: unknown op %d", fn, op);
      return 0;
  }
}

rswa_status rswa_check_status(void* workspace, size_t ws_bytes, int32_t* device_status, void* stream) {
  const char* fn = "rswa_check_status";
  if (workspace == nullptr || ws_bytes < 4) return fail(RSWA_ERR_INVALID, "%s: workspace must hold the status word", fn);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t host = 0;
  cudaError_t e = cudaMemcpyAsync(&host, workspace, sizeof host, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "rswa_check_status: reading the status word");
  if (host != 0) {
    // a timed-out wait can leave completion counters of the abandoned work items behind: the
    // whole workspace goes back to its zero-filled initial state; otherwise only the status word
    const size_t clear = (host & RSWA_DEVICE_WAIT_TIMEOUT) ? ws_bytes : sizeof(int32_t);
    e = cudaMemsetAsync(workspace, 0, clear, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e, "rswa_check_status: clearing the status word");
  }
  if (device_status) *device_status = host;
  if (host != 0) return fail(RSWA_ERR_DEVICE_CHECK, "%s: device status 0x%x", fn, host);
  return ok();
}

rswa_status rswa_test_arm_wait_timeout(int32_t drop_tile, int64_t wait_limit_ns) {
  const char* fn = "rswa_test_arm_wait_timeout";
  if (drop_tile < -1) return fail(RSWA_ERR_INVALID, "%s: drop_tile must be >= -1 (got %d)", fn, drop_tile);
  if (wait_limit_ns < 1000 || wait_limit_ns > 10000000000ll)
    return fail(RSWA_ERR_INVALID, "%s: wait_limit_ns must be in [1e3, 1e10] (got %lld)", fn, (long long)wait_limit_ns);
  g_test_drop_tile = drop_tile;
  g_test_wait_ns = (uint64_t)wait_limit_ns;
  return ok();
}

rswa_status rswa_append(const rswa_dims* dims, void* ring_k, void* ring_v, const void* k_new, const void* v_new,
                        int32_t* wp, int32_t* fill, int32_t* slot_out, int32_t* status, void* stream) {
  const char* fn = "rswa_append";
  const NvtxRange nvtx_range(fn);
  rswa_status st = check_dims(fn, dims, false);
  if (st != RSWA_OK) return st;
  REQUIRE_PTR(ring_k);
  REQUIRE_PTR(ring_v);
  REQUIRE_PTR(k_new);
  REQUIRE_PTR(v_new);
  if (wp == nullptr || fill == nullptr) return fail(RSWA_ERR_INVALID, "%s: wp and fill must not be NULL", fn);
  cudaError_t e = rswa::launch_append(dims->batch, dims->heads, dims->ring, static_cast<uint16_t*>(ring_k),
                                      static_cast<uint16_t*>(ring_v), static_cast<const uint16_t*>(k_new),
                                      static_cast<const uint16_t*>(v_new), wp, fill, slot_out, status,
                                      static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "rswa_append: launch");
  return ok();
}

// The prefix K/V of a decode call: bf16 rows, or E4M3 code rows with block scales.
struct PrefixSrc {
  const void* k;
  const void* v;
  const float* ks;
  const float* vs;
  bool fp8;
};

static PrefixSrc bf16_prefix(const void* pk, const void* pv) { return PrefixSrc{pk, pv, nullptr, nullptr, false}; }

// SR-SWA chunked prefill: T queries per (sequence, head) whose causal band is read from the
// chunk's output K/V; T = 1 and no band for decode.
struct BandSrc {
  int T;
  const void* k_out;
  const void* v_out;
};
constexpr BandSrc kNoBand{1, nullptr, nullptr};

// Fused ring append: this step's K / V join the ring inside the decode launch.
struct AppendSrc {
  const void* k_new;
  const void* v_new;
  void* ring_k;  // the same ring as the decode reads, writable
  void* ring_v;
  int32_t* wp;
  int32_t* fill;
  int32_t* slot_out;
  const rswa_rope* rope;  // page2d encoding of this step's query and key, or null
};
constexpr AppendSrc kNoAppend{nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr};

// An FP8 ring (codes + row scales) in place of the bf16 ring_k / ring_v.
struct Ring8Src {
  const void* k8;
  const void* v8;
  const float* ks;
  const float* vs;
  bool on;
};
constexpr Ring8Src kNoRing8{nullptr, nullptr, nullptr, nullptr, false};

// The SR-SWA router fused into the decode launch: its inputs and the route outputs.
struct RouteSrc {
  const float* q_idx;
  const float* kbar;
  float idx_scale;
  int32_t* blk_idx;
  float* blk_logp;
  float* tau;
  bool on;
};
constexpr RouteSrc kNoRoute{nullptr, nullptr, 0.f, nullptr, nullptr, nullptr, false};
constexpr size_t kGridCounterOffset = 128;  // an int32 inside the workspace's 256-byte status area

// page2d rotary encoding: the checks shared by the entry points that encode.
static rswa_status check_rope_params(const char* fn, const int32_t* tok_pos, const int32_t* page, double base,
                                     int32_t page_mod) {
  if (tok_pos == nullptr || page == nullptr) return fail(RSWA_ERR_INVALID, "%s: tok_pos and page must not be NULL", fn);
  if (!(base > 0.0) || !std::isfinite(base)) return fail(RSWA_ERR_INVALID, "%s: base must be finite and > 0", fn);
  if (page_mod < 0) return fail(RSWA_ERR_INVALID, "%s: page_mod must be >= 0 (got %d)", fn, page_mod);
  return RSWA_OK;
}

// plan_budget > 0: plan the split-KV work to fit a workspace of that many bytes.
static rswa_status decode_common(const char* fn, bool sparse, const rswa_dims* dims, const void* q, PrefixSrc px,
                                 BandSrc band, AppendSrc app, const int32_t* prefix_len, const int32_t* blk_idx,
                                 const float* blk_logp, int32_t topk, const void* ring_k, const void* ring_v,
                                 const int32_t* wp, const int32_t* fill, float scale, float* out, float* lse,
                                 void* workspace, size_t ws_bytes, void* stream, size_t plan_budget = 0,
                                 Ring8Src r8 = kNoRing8, RouteSrc rt = kNoRoute) {
  const NvtxRange nvtx_range(fn);
  // a wait-timeout test knob applies to this call only, whether or not it launches
  const int test_drop_tile = g_test_drop_tile;
  const uint64_t test_wait_ns = g_test_wait_ns;
  g_test_drop_tile = -1;
  g_test_wait_ns = 0;
  rswa_status st = check_dims(fn, dims, true);
  if (st != RSWA_OK) return st;
  REQUIRE_PTR(q);
  const void* pk = px.k;
  const void* pv = px.v;
  REQUIRE_PTR(pk);
  REQUIRE_PTR(pv);
  if (px.fp8) {
    const float* k_scale = px.ks;
    const float* v_scale = px.vs;
    REQUIRE_PTR(k_scale);
    REQUIRE_PTR(v_scale);
  }
  const bool prefill = band.k_out != nullptr;
  if (prefill) {  // the ring (the previous chunk) is optional
    const void* k_out = band.k_out;
    const void* v_out = band.v_out;
    REQUIRE_PTR(k_out);
    REQUIRE_PTR(v_out);
    if (band.T < 1) return fail(RSWA_ERR_INVALID, "%s: T must be >= 1 (got %d)", fn, band.T);
    if ((ring_k == nullptr) != (ring_v == nullptr))
      return fail(RSWA_ERR_INVALID, "%s: ring_k and ring_v must both be given or both be NULL", fn);
    if (ring_k != nullptr && (wp == nullptr || fill == nullptr))
      return fail(RSWA_ERR_INVALID, "%s: a ring needs wp and fill", fn);
    REQUIRE_PTR_OR_NULL(ring_k);
    REQUIRE_PTR_OR_NULL(ring_v);
    if (prefix_len == nullptr) return fail(RSWA_ERR_INVALID, "%s: prefix_len must not be NULL", fn);
  } else if (r8.on) {
    const void* ring_k8 = r8.k8;
    const void* ring_v8 = r8.v8;
    const float* ring_kscale = r8.ks;
    const float* ring_vscale = r8.vs;
    REQUIRE_PTR(ring_k8);
    REQUIRE_PTR(ring_v8);
    REQUIRE_PTR(ring_kscale);
    REQUIRE_PTR(ring_vscale);
    if (!px.fp8) return fail(RSWA_ERR_UNSUPPORTED, "%s: an FP8 ring needs an FP8 prefix", fn);
    if (prefix_len == nullptr || wp == nullptr || fill == nullptr)
      return fail(RSWA_ERR_INVALID, "%s: prefix_len, wp and fill must not be NULL", fn);
  } else {
    REQUIRE_PTR(ring_k);
    REQUIRE_PTR(ring_v);
    if (prefix_len == nullptr || wp == nullptr || fill == nullptr)
      return fail(RSWA_ERR_INVALID, "%s: prefix_len, wp and fill must not be NULL", fn);
  }
  REQUIRE_PTR(out);
  REQUIRE_PTR(workspace);
  if (app.k_new != nullptr) {
    const void* k_new = app.k_new;
    const void* v_new = app.v_new;
    REQUIRE_PTR(k_new);
    REQUIRE_PTR(v_new);
    if (app.rope != nullptr) {
      st = check_rope_params(fn, app.rope->tok_pos, app.rope->page, app.rope->base, app.rope->page_mod);
      if (st != RSWA_OK) return st;
    }
  }
  if (sparse) {
    if (blk_idx == nullptr || blk_logp == nullptr)
      return fail(RSWA_ERR_INVALID, "%s: blk_idx and blk_logp must not be NULL", fn);
    if (topk < 1 || topk > rswa::kMaxTopk) return fail(RSWA_ERR_INVALID, "%s: topk must be in [1, 32] (got %d)", fn, topk);
  }
  if (rt.on) {
    const float* q_idx = rt.q_idx;
    const float* kbar = rt.kbar;
    REQUIRE_PTR(q_idx);
    REQUIRE_PTR(kbar);
    if (!std::isfinite(rt.idx_scale)) return fail(RSWA_ERR_INVALID, "%s: idx_scale must be finite", fn);
    const int64_t nb_cap = (dims->prefix_cap + rswa::kBlock - 1) / rswa::kBlock;
    if (nb_cap == 0) return fail(RSWA_ERR_INVALID, "%s: prefix_cap must be >= 1", fn);
    if (nb_cap > rswa::kMaxRouteBlocks)
      return fail(RSWA_ERR_UNSUPPORTED, "%s: %lld prefix blocks exceed the router's limit of %d", fn,
                  (long long)nb_cap, rswa::kMaxRouteBlocks);
  }
  if (!(scale > 0.f) || !std::isfinite(scale)) return fail(RSWA_ERR_INVALID, "%s: scale must be finite and > 0", fn);
  int64_t max_tiles = sparse ? rswa::decode_max_tiles_sparse(topk, dims->ring)
                             : rswa::decode_max_tiles_dense(dims->prefix_cap, dims->ring);
  if (app.k_new != nullptr) max_tiles += 1;  // this step's token
  rswa::WorkspacePlan plan;
  if (prefill) {
    // ring part and band together cover n keys in at most three ranges: two tiles beyond a decode's
    max_tiles += 2;
    const int64_t queries = (int64_t)dims->batch * dims->heads * band.T;
    if (queries > INT32_MAX) return fail(RSWA_ERR_UNSUPPORTED, "%s: too many queries", fn);
    // many queries: one split each (the status word is all the workspace needed)
    const int64_t slots = (int64_t)rswa::device_sm_count() * rswa::decode_ctas_per_sm();
    plan.splits = 1;
    plan.tiles_per_item = (int)max_tiles;
    plan.items = queries;
    plan.grid = (int)(queries < slots ? queries : slots);
    plan.counters_off = plan.partials_off = 0;
    plan.bytes = 256;
  } else {
    plan = rswa::plan_decode_workspace(dims->batch, dims->heads, max_tiles, rswa::device_sm_count(), plan_budget);
  }
  size_t need = plan.bytes, route_off = 0;
  int n_fin = 0;
  if (rt.on) {
    // the fused router's CTAs wait on one another: the grid must fit one resident wave of this
    // kernel, and its last CTAs (item-free when there is room) finalise the routes
    const int per_sm = rswa::routed_decode_ctas_per_sm();
    if (per_sm < 1) return fail(RSWA_ERR_CUDA, "%s: occupancy query of the fused router kernel failed", fn);
    const int64_t slots = (int64_t)rswa::device_sm_count() * per_sm;
    const int64_t want = plan.items + dims->batch;
    plan.grid = (int)(want < slots ? want : slots);
    n_fin = dims->batch < plan.grid ? dims->batch : plan.grid;
    route_off = align256(plan.bytes);
    need = route_off + rswa::route_area_bytes(dims->batch, dims->prefix_cap);
  }
  if (ws_bytes < need)
    return fail(RSWA_ERR_INVALID, "%s: workspace of %zu bytes is smaller than the %zu required", fn, ws_bytes, need);
  rswa::DecodeArgs a;
  a.B = dims->batch;
  a.H = dims->heads;
  a.n = dims->ring;
  a.cap = dims->prefix_cap;
  a.splits = plan.splits;
  a.tiles_per_item = plan.tiles_per_item;
  if (plan.items > INT32_MAX) return fail(RSWA_ERR_UNSUPPORTED, "%s: too many work items", fn);
  a.items = (int)plan.items;
  a.q = static_cast<const uint16_t*>(q);
  a.fp8 = px.fp8 ? 1 : 0;
  a.pk = px.fp8 ? nullptr : static_cast<const uint16_t*>(pk);
  a.pv = px.fp8 ? nullptr : static_cast<const uint16_t*>(pv);
  a.pk8 = px.fp8 ? static_cast<const uint8_t*>(pk) : nullptr;
  a.pv8 = px.fp8 ? static_cast<const uint8_t*>(pv) : nullptr;
  a.kscale = px.ks;
  a.vscale = px.vs;
  a.nb_cap = (dims->prefix_cap + rswa::kBlock - 1) / rswa::kBlock;
  a.T = prefill ? band.T : 1;
  a.k_out = static_cast<const uint16_t*>(band.k_out);
  a.v_out = static_cast<const uint16_t*>(band.v_out);
  a.k_new = static_cast<const uint16_t*>(app.k_new);
  a.v_new = static_cast<const uint16_t*>(app.v_new);
  a.ring_k_w = static_cast<uint16_t*>(app.ring_k);
  a.ring_v_w = static_cast<uint16_t*>(app.ring_v);
  a.wp_w = app.wp;
  a.fill_w = app.fill;
  a.slot_out = app.slot_out;
  a.rope_tok = app.rope ? app.rope->tok_pos : nullptr;
  a.rope_page = app.rope ? app.rope->page : nullptr;
  a.rope_log2_base = app.rope ? std::log2(app.rope->base) : 0.0;
  a.rope_page_mod = app.rope ? app.rope->page_mod : 0;
  a.grid_counter = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(workspace) + kGridCounterOffset);
  a.prefix_len = prefix_len;
  a.ring_k = static_cast<const uint16_t*>(ring_k);
  a.ring_v = static_cast<const uint16_t*>(ring_v);
  a.ring_k8 = static_cast<const uint8_t*>(r8.k8);
  a.ring_v8 = static_cast<const uint8_t*>(r8.v8);
  a.ring_ks = r8.ks;
  a.ring_vs = r8.vs;
  a.wp = wp;
  a.fill = fill;
  a.qscale = scale * 1.4426950408889634f;
  a.out = out;
  a.lse = lse;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  a.status = ws_status(workspace);
  a.counters = prefill ? nullptr : reinterpret_cast<int32_t*>(ws + plan.counters_off);
  a.partials = prefill ? nullptr : reinterpret_cast<float*>(ws + plan.partials_off);
  a.blk_idx = blk_idx;
  a.blk_logp = blk_logp;
  a.topk = sparse ? topk : 0;
  a.wait_limit_ns = test_wait_ns > 0 ? test_wait_ns : rswa::kWaitLimitNs;
  a.drop_tile = test_drop_tile;
  a.q_idx = rt.q_idx;
  a.kbar = rt.kbar;
  a.idx_scale = rt.idx_scale;
  a.nsl_cap = (int)(((dims->prefix_cap + rswa::kBlock - 1) / rswa::kBlock + 63) / 64);
  a.n_fin = n_fin;
  a.blk_idx_w = rt.blk_idx;
  a.blk_logp_w = rt.blk_logp;
  a.tau_w = rt.tau;
  a.seq_count = a.route_ready = nullptr;
  a.slice_max = a.slice_z = nullptr;
  a.slice_i = nullptr;
  if (rt.on) {  // route area: [seq_count, route_ready][slice_max][slice_z][slice_i]
    uint8_t* r = ws + route_off;
    const size_t B = (size_t)dims->batch, nsl = (size_t)a.nsl_cap;
    a.seq_count = reinterpret_cast<int32_t*>(r);
    a.route_ready = a.seq_count + B;
    r += align256(B * 8);
    a.slice_max = reinterpret_cast<float*>(r);
    r += align256(B * nsl * 4);
    a.slice_z = reinterpret_cast<float*>(r);
    a.slice_i = reinterpret_cast<int32_t*>(a.slice_z + B * nsl * 64);
  }
  cudaError_t e = rswa::launch_decode(a, plan.grid, sparse, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, fn);
  return ok();
}

rswa_status rswa_decode(const rswa_dims* dims, const void* q, const void* pk, const void* pv,
                        const int32_t* prefix_len, const void* ring_k, const void* ring_v, const int32_t* wp,
                        const int32_t* fill, float scale, float* out, float* lse, void* workspace, size_t ws_bytes,
                        void* stream) {
  return decode_common("rswa_decode", false, dims, q, bf16_prefix(pk, pv), kNoBand, kNoAppend, prefix_len, nullptr,
                       nullptr, 0, ring_k,
                       ring_v, wp, fill, scale, out, lse, workspace, ws_bytes, stream);
}

rswa_status rswa_decode_fp8(const rswa_dims* dims, const void* q, const uint8_t* pk8, const uint8_t* pv8,
                            const float* k_scale, const float* v_scale, const int32_t* prefix_len, const void* ring_k,
                            const void* ring_v, const int32_t* wp, const int32_t* fill, float scale, float* out,
                            float* lse, void* workspace, size_t ws_bytes, void* stream) {
  return decode_common("rswa_decode_fp8", false, dims, q, PrefixSrc{pk8, pv8, k_scale, v_scale, true}, kNoBand,
                       kNoAppend, prefix_len,
                       nullptr, nullptr, 0, ring_k, ring_v, wp, fill, scale, out, lse, workspace, ws_bytes, stream);
}

rswa_status srswa_decode_fp8(const rswa_dims* dims, const void* q, const uint8_t* pk8, const uint8_t* pv8,
                             const float* k_scale, const float* v_scale, const int32_t* prefix_len,
                             const int32_t* blk_idx, const float* blk_logp, int32_t topk, const void* ring_k,
                             const void* ring_v, const int32_t* wp, const int32_t* fill, float scale, float* out,
                             float* lse, void* workspace, size_t ws_bytes, void* stream) {
  return decode_common("srswa_decode_fp8", true, dims, q, PrefixSrc{pk8, pv8, k_scale, v_scale, true}, kNoBand,
                       kNoAppend, prefix_len,
                       blk_idx, blk_logp, topk, ring_k, ring_v, wp, fill, scale, out, lse, workspace, ws_bytes, stream);
}

rswa_status rswa_decode_fp8kv(const rswa_dims* dims, const void* q, const uint8_t* pk8, const uint8_t* pv8,
                              const float* k_scale, const float* v_scale, const int32_t* prefix_len,
                              const uint8_t* ring_k8, const uint8_t* ring_v8, const float* ring_kscale,
                              const float* ring_vscale, const int32_t* wp, const int32_t* fill, float scale, float* out,
                              float* lse, void* workspace, size_t ws_bytes, void* stream) {
  return decode_common("rswa_decode_fp8kv", false, dims, q, PrefixSrc{pk8, pv8, k_scale, v_scale, true}, kNoBand,
                       kNoAppend, prefix_len, nullptr, nullptr, 0, nullptr, nullptr, wp, fill, scale, out, lse,
                       workspace, ws_bytes, stream, 0, Ring8Src{ring_k8, ring_v8, ring_kscale, ring_vscale, true});
}

rswa_status srswa_decode_fp8kv(const rswa_dims* dims, const void* q, const uint8_t* pk8, const uint8_t* pv8,
                               const float* k_scale, const float* v_scale, const int32_t* prefix_len,
                               const int32_t* blk_idx, const float* blk_logp, int32_t topk, const uint8_t* ring_k8,
                               const uint8_t* ring_v8, const float* ring_kscale, const float* ring_vscale,
                               const int32_t* wp, const int32_t* fill, float scale, float* out, float* lse,
                               void* workspace, size_t ws_bytes, void* stream) {
  return decode_common("srswa_decode_fp8kv", true, dims, q, PrefixSrc{pk8, pv8, k_scale, v_scale, true}, kNoBand,
                       kNoAppend, prefix_len, blk_idx, blk_logp, topk, nullptr, nullptr, wp, fill, scale, out, lse,
                       workspace, ws_bytes, stream, 0, Ring8Src{ring_k8, ring_v8, ring_kscale, ring_vscale, true});
}

rswa_status rswa_append_fp8(const rswa_dims* dims, uint8_t* ring_k8, uint8_t* ring_v8, float* ring_kscale,
                            float* ring_vscale, const void* k_new, const void* v_new, int32_t* wp, int32_t* fill,
                            int32_t* slot_out, int32_t* status, void* stream) {
  const char* fn = "rswa_append_fp8";
  const NvtxRange nvtx_range(fn);
  rswa_status st = check_dims(fn, dims, false);
  if (st != RSWA_OK) return st;
  REQUIRE_PTR(ring_k8);
  REQUIRE_PTR(ring_v8);
  REQUIRE_PTR(ring_kscale);
  REQUIRE_PTR(ring_vscale);
  REQUIRE_PTR(k_new);
  REQUIRE_PTR(v_new);
  if (wp == nullptr || fill == nullptr) return fail(RSWA_ERR_INVALID, "%s: wp and fill must not be NULL", fn);
  cudaError_t e = rswa::launch_append_fp8(dims->batch, dims->heads, dims->ring, ring_k8, ring_v8, ring_kscale,
                                          ring_vscale, static_cast<const uint16_t*>(k_new),
                                          static_cast<const uint16_t*>(v_new), wp, fill, slot_out, status,
                                          static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, fn);
  return ok();
}

rswa_status rswa_quantize_prefix(const rswa_dims* dims, const void* pk, const void* pv, const int32_t* prefix_len,
                                 uint8_t* pk8, uint8_t* pv8, float* k_scale, float* v_scale, int32_t* status,
                                 void* stream) {
  const char* fn = "rswa_quantize_prefix";
  const NvtxRange nvtx_range(fn);
  rswa_status st = check_dims(fn, dims, true);
  if (st != RSWA_OK) return st;
  REQUIRE_PTR(pk);
  REQUIRE_PTR(pv);
  REQUIRE_PTR(pk8);
  REQUIRE_PTR(pv8);
  REQUIRE_PTR(k_scale);
  REQUIRE_PTR(v_scale);
  if (prefix_len == nullptr) return fail(RSWA_ERR_INVALID, "%s: prefix_len must not be NULL", fn);
  if ((int64_t)dims->batch * dims->heads > 65535)
    return fail(RSWA_ERR_UNSUPPORTED, "%s: batch * heads above 65535", fn);
  cudaError_t e = rswa::launch_quantize_prefix(dims->batch, dims->heads, dims->prefix_cap,
                                               static_cast<const uint16_t*>(pk), static_cast<const uint16_t*>(pv),
                                               prefix_len, pk8, pv8, k_scale, v_scale, status,
                                               static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, fn);
  return ok();
}

rswa_status rswa_rope_page2d(int64_t rows, int32_t heads, int32_t head_dim, const void* q, void* q_out, const void* k,
                             void* k_out, const int32_t* tok_pos, const int32_t* page, double base, int32_t page_mod,
                             void* stream) {
  const char* fn = "rswa_rope_page2d";
  const NvtxRange nvtx_range(fn);
  if (rows < 0) return fail(RSWA_ERR_INVALID, "%s: rows must be >= 0 (got %lld)", fn, (long long)rows);
  if (heads < 1 || heads > 128) return fail(RSWA_ERR_INVALID, "%s: heads must be in [1, 128] (got %d)", fn, heads);
  if (head_dim < 16 || head_dim > 256 || head_dim % 16 != 0)
    return fail(RSWA_ERR_UNSUPPORTED, "%s: head_dim must be a multiple of 16 in [16, 256] (got %d)", fn, head_dim);
  if (!(base > 0.0) || !std::isfinite(base)) return fail(RSWA_ERR_INVALID, "%s: base must be finite and > 0", fn);
  if (page_mod < 0) return fail(RSWA_ERR_INVALID, "%s: page_mod must be >= 0 (got %d)", fn, page_mod);
  if (rows == 0) return ok();  // nothing to encode; the (empty) buffers may be NULL
  REQUIRE_PTR(q);
  REQUIRE_PTR(q_out);
  if ((k == nullptr) != (k_out == nullptr)) return fail(RSWA_ERR_INVALID, "%s: k and k_out must both be given or both NULL", fn);
  REQUIRE_PTR_OR_NULL(k);
  REQUIRE_PTR_OR_NULL(k_out);
  rswa_status st = check_rope_params(fn, tok_pos, page, base, page_mod);
  if (st != RSWA_OK) return st;
  cudaError_t e = rswa::launch_rope(rows, heads, head_dim, static_cast<const uint16_t*>(q), static_cast<uint16_t*>(q_out),
                                    static_cast<const uint16_t*>(k), static_cast<uint16_t*>(k_out), tok_pos, page, base,
                                    page_mod, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, fn);
  return ok();
}

rswa_status rswa_append_rope(const rswa_dims* dims, void* ring_k, void* ring_v, const void* k_new, const void* v_new,
                             int32_t* wp, int32_t* fill, int32_t* slot_out, const void* q, void* q_out,
                             const int32_t* tok_pos, const int32_t* page, double base, int32_t page_mod, int32_t* status,
                             void* stream) {
  const char* fn = "rswa_append_rope";
  const NvtxRange nvtx_range(fn);
  rswa_status st = check_dims(fn, dims, false);
  if (st != RSWA_OK) return st;
  REQUIRE_PTR(ring_k);
  REQUIRE_PTR(ring_v);
  REQUIRE_PTR(k_new);
  REQUIRE_PTR(v_new);
  REQUIRE_PTR(q);
  REQUIRE_PTR(q_out);
  if (wp == nullptr || fill == nullptr) return fail(RSWA_ERR_INVALID, "%s: wp and fill must not be NULL", fn);
  st = check_rope_params(fn, tok_pos, page, base, page_mod);
  if (st != RSWA_OK) return st;
  cudaError_t e = rswa::launch_append_rope(
      dims->batch, dims->heads, dims->ring, static_cast<uint16_t*>(ring_k), static_cast<uint16_t*>(ring_v),
      static_cast<const uint16_t*>(k_new), static_cast<const uint16_t*>(v_new), static_cast<const uint16_t*>(q),
      static_cast<uint16_t*>(q_out), tok_pos, page, base, page_mod, wp, fill, slot_out, status,
      static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, fn);
  return ok();
}

rswa_status srswa_decode(const rswa_dims* dims, const void* q, const void* pk, const void* pv,
                         const int32_t* prefix_len, const int32_t* blk_idx, const float* blk_logp, int32_t topk,
                         const void* ring_k, const void* ring_v, const int32_t* wp, const int32_t* fill, float scale,
                         float* out, float* lse, void* workspace, size_t ws_bytes, void* stream) {
  return decode_common("srswa_decode", true, dims, q, bf16_prefix(pk, pv), kNoBand, kNoAppend, prefix_len, blk_idx,
                       blk_logp, topk, ring_k,
                       ring_v, wp, fill, scale, out, lse, workspace, ws_bytes, stream);
}

rswa_status rswa_decode_append(const rswa_dims* dims, const void* q, const void* k_new, const void* v_new,
                               const void* pk, const void* pv, const int32_t* prefix_len, void* ring_k, void* ring_v,
                               int32_t* wp, int32_t* fill, int32_t* slot_out, float scale, float* out, float* lse,
                               void* workspace, size_t ws_bytes, void* stream) {
  if (k_new == nullptr || v_new == nullptr)
    return fail(RSWA_ERR_INVALID, "rswa_decode_append: k_new and v_new must not be NULL");
  return decode_common("rswa_decode_append", false, dims, q, bf16_prefix(pk, pv), kNoBand,
                       AppendSrc{k_new, v_new, ring_k, ring_v, wp, fill, slot_out, nullptr}, prefix_len, nullptr,
                       nullptr, 0, ring_k, ring_v, wp, fill, scale, out, lse, workspace, ws_bytes, stream);
}

rswa_status srswa_decode_append(const rswa_dims* dims, const void* q, const void* k_new, const void* v_new,
                                const void* pk, const void* pv, const int32_t* prefix_len, const int32_t* blk_idx,
                                const float* blk_logp, int32_t topk, void* ring_k, void* ring_v, int32_t* wp,
                                int32_t* fill, int32_t* slot_out, float scale, float* out, float* lse,
                                void* workspace, size_t ws_bytes, void* stream) {
  if (k_new == nullptr || v_new == nullptr)
    return fail(RSWA_ERR_INVALID, "srswa_decode_append: k_new and v_new must not be NULL");
  return decode_common("srswa_decode_append", true, dims, q, bf16_prefix(pk, pv), kNoBand,
                       AppendSrc{k_new, v_new, ring_k, ring_v, wp, fill, slot_out, nullptr}, prefix_len, blk_idx,
                       blk_logp, topk, ring_k, ring_v, wp, fill, scale, out, lse, workspace, ws_bytes, stream);
}

rswa_status srswa_decode_routed(const rswa_dims* dims, const void* q, const float* q_idx, const float* kbar,
                                float idx_scale, int32_t topk, const void* pk, const void* pv,
                                const int32_t* prefix_len, const void* ring_k, const void* ring_v, const int32_t* wp,
                                const int32_t* fill, float scale, int32_t* blk_idx, float* blk_logp, float* tau,
                                float* out, float* lse, void* workspace, size_t ws_bytes, void* stream) {
  return decode_common("srswa_decode_routed", true, dims, q, bf16_prefix(pk, pv), kNoBand, kNoAppend, prefix_len,
                       blk_idx, blk_logp, topk, ring_k, ring_v, wp, fill, scale, out, lse, workspace, ws_bytes,
                       stream, 0, kNoRing8, RouteSrc{q_idx, kbar, idx_scale, blk_idx, blk_logp, tau, true});
}

rswa_status srswa_step(const rswa_dims* dims, const void* q, const void* k_new, const void* v_new, const float* q_idx,
                       const float* kbar, float idx_scale, int32_t topk, const void* pk, const void* pv,
                       const int32_t* prefix_len, void* ring_k, void* ring_v, int32_t* wp, int32_t* fill,
                       int32_t* slot_out, float scale, int32_t* blk_idx, float* blk_logp, float* tau, float* out,
                       float* lse, void* workspace, size_t ws_bytes, void* stream) {
  if (k_new == nullptr || v_new == nullptr) return fail(RSWA_ERR_INVALID, "srswa_step: k_new and v_new must not be NULL");
  return decode_common("srswa_step", true, dims, q, bf16_prefix(pk, pv), kNoBand,
                       AppendSrc{k_new, v_new, ring_k, ring_v, wp, fill, slot_out, nullptr}, prefix_len, blk_idx,
                       blk_logp, topk, ring_k, ring_v, wp, fill, scale, out, lse, workspace, ws_bytes, stream, 0,
                       kNoRing8, RouteSrc{q_idx, kbar, idx_scale, blk_idx, blk_logp, tau, true});
}

rswa_status rswa_decode_append_rope(const rswa_dims* dims, const rswa_rope* rope, const void* q, const void* k_new,
                                    const void* v_new, const void* pk, const void* pv, const int32_t* prefix_len,
                                    void* ring_k, void* ring_v, int32_t* wp, int32_t* fill, int32_t* slot_out,
                                    float scale, float* out, float* lse, void* workspace, size_t ws_bytes,
                                    void* stream) {
  const char* fn = "rswa_decode_append_rope";
  if (rope == nullptr) return fail(RSWA_ERR_INVALID, "%s: rope must not be NULL", fn);
  if (k_new == nullptr || v_new == nullptr) return fail(RSWA_ERR_INVALID, "%s: k_new and v_new must not be NULL", fn);
  return decode_common(fn, false, dims, q, bf16_prefix(pk, pv), kNoBand,
                       AppendSrc{k_new, v_new, ring_k, ring_v, wp, fill, slot_out, rope}, prefix_len, nullptr, nullptr,
                       0, ring_k, ring_v, wp, fill, scale, out, lse, workspace, ws_bytes, stream);
}

rswa_status srswa_step_rope(const rswa_dims* dims, const rswa_rope* rope, const void* q, const void* k_new,
                            const void* v_new, const float* q_idx, const float* kbar, float idx_scale, int32_t topk,
                            const void* pk, const void* pv, const int32_t* prefix_len, void* ring_k, void* ring_v,
                            int32_t* wp, int32_t* fill, int32_t* slot_out, float scale, int32_t* blk_idx,
                            float* blk_logp, float* tau, float* out, float* lse, void* workspace, size_t ws_bytes,
                            void* stream) {
  const char* fn = "srswa_step_rope";
  if (rope == nullptr) return fail(RSWA_ERR_INVALID, "%s: rope must not be NULL", fn);
  if (k_new == nullptr || v_new == nullptr) return fail(RSWA_ERR_INVALID, "%s: k_new and v_new must not be NULL", fn);
  return decode_common(fn, true, dims, q, bf16_prefix(pk, pv), kNoBand,
                       AppendSrc{k_new, v_new, ring_k, ring_v, wp, fill, slot_out, rope}, prefix_len, blk_idx,
                       blk_logp, topk, ring_k, ring_v, wp, fill, scale, out, lse, workspace, ws_bytes, stream, 0,
                       kNoRing8, RouteSrc{q_idx, kbar, idx_scale, blk_idx, blk_logp, tau, true});
}

rswa_status rswa_prefill(const rswa_dims* dims, int32_t T, const void* q, const void* k_out, const void* v_out,
                         const void* pk, const void* pv, const int32_t* prefix_len, void* ring_k, void* ring_v,
                         int32_t* wp, int32_t* fill, float scale, float* out, float* lse, int32_t write_ring,
                         void* workspace, size_t ws_bytes, void* stream) {
  const char* fn = "rswa_prefill";
  const NvtxRange nvtx_range(fn);
  rswa_status st = check_dims(fn, dims, true);
  if (st != RSWA_OK) return st;
  if (T < 1) return fail(RSWA_ERR_INVALID, "%s: T must be >= 1 (got %d)", fn, T);
  REQUIRE_PTR(q);
  REQUIRE_PTR(k_out);
  REQUIRE_PTR(v_out);
  REQUIRE_PTR(out);
  REQUIRE_PTR(workspace);
  REQUIRE_PTR_OR_NULL(lse);
  if (prefix_len == nullptr) return fail(RSWA_ERR_INVALID, "%s: prefix_len must not be NULL", fn);
  if (dims->prefix_cap > 0) {
    REQUIRE_PTR(pk);
    REQUIRE_PTR(pv);
  }
  const bool ring = ring_k != nullptr || ring_v != nullptr || wp != nullptr || fill != nullptr;
  if (ring) {
    REQUIRE_PTR(ring_k);
    REQUIRE_PTR(ring_v);
    if (wp == nullptr || fill == nullptr) return fail(RSWA_ERR_INVALID, "%s: a ring needs wp and fill", fn);
  } else if (write_ring) {
    return fail(RSWA_ERR_INVALID, "%s: write_ring needs a ring", fn);
  }
  if (!(scale > 0.f) || !std::isfinite(scale)) return fail(RSWA_ERR_INVALID, "%s: scale must be finite and > 0", fn);
  if (ws_bytes < 256) return fail(RSWA_ERR_INVALID, "%s: workspace must be at least 256 bytes", fn);
  const int64_t bh = (int64_t)dims->batch * dims->heads;
  const int64_t lim = ((int64_t)1 << 31) - 1;
  if (bh * T >= lim || bh * dims->prefix_cap >= lim || bh * dims->ring >= lim)
    return fail(RSWA_ERR_UNSUPPORTED, "%s: more than 2^31 rows in one operand", fn);
  rswa::PrefillLaunch L;
  L.B = dims->batch;
  L.H = dims->heads;
  L.n = dims->ring;
  L.T = T;
  L.cap = dims->prefix_cap;
  L.q = q;
  L.k_out = k_out;
  L.v_out = v_out;
  L.pk = pk;
  L.pv = pv;
  L.prefix_len = prefix_len;
  L.ring_k = ring ? ring_k : nullptr;
  L.ring_v = ring ? ring_v : nullptr;
  L.wp = wp;
  L.fill = fill;
  L.scale = scale;
  L.out = out;
  L.lse = lse;
  L.write_ring = write_ring ? 1 : 0;
  L.ring_k_w = ring_k;
  L.ring_v_w = ring_v;
  L.wp_w = wp;
  L.fill_w = fill;
  L.status = ws_status(workspace);
  L.ignore_prefix = 0;
  cudaError_t e = rswa::launch_prefill(L, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, fn);
  return ok();
}

rswa_status srswa_index_pool(const rswa_dims* dims, const void* k_idx, const int32_t* prefix_len, float* kbar,
                             void* stream) {
  const char* fn = "srswa_index_pool";
  const NvtxRange nvtx_range(fn);
  rswa_status st = check_dims(fn, dims, true);
  if (st != RSWA_OK) return st;
  REQUIRE_PTR(k_idx);
  REQUIRE_PTR(kbar);
  if (prefix_len == nullptr) return fail(RSWA_ERR_INVALID, "%s: prefix_len must not be NULL", fn);
  if (dims->prefix_cap == 0) return ok();
  cudaError_t e = rswa::launch_index_pool(dims->batch, dims->prefix_cap, static_cast<const uint16_t*>(k_idx),
                                          prefix_len, kbar, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, fn);
  return ok();
}

static rswa_status route_common(const char* fn, const rswa_dims* dims, int tokens, const float* q_idx,
                                const float* kbar, const int32_t* prefix_len, float idx_scale, int32_t topk,
                                int32_t* blk_idx, float* blk_logp, float* probs, float* tau, void* workspace,
                                size_t ws_bytes, void* stream) {
  const NvtxRange nvtx_range(fn);
  rswa_status st = check_dims(fn, dims, true);
  if (st != RSWA_OK) return st;
  REQUIRE_PTR(q_idx);
  REQUIRE_PTR(kbar);
  REQUIRE_PTR(workspace);
  REQUIRE_PTR_OR_NULL(probs);
  if (prefix_len == nullptr || blk_idx == nullptr || blk_logp == nullptr)
    return fail(RSWA_ERR_INVALID, "%s: prefix_len, blk_idx and blk_logp must not be NULL", fn);
  if (topk < 1 || topk > rswa::kMaxTopk) return fail(RSWA_ERR_INVALID, "%s: topk must be in [1, 32] (got %d)", fn, topk);
  if (!std::isfinite(idx_scale)) return fail(RSWA_ERR_INVALID, "%s: idx_scale must be finite", fn);
  if (tokens < 1) return fail(RSWA_ERR_INVALID, "%s: T must be >= 1 (got %d)", fn, tokens);
  if ((int64_t)dims->batch * tokens > 65535)
    return fail(RSWA_ERR_UNSUPPORTED, "%s: batch * T above 65535 router queries", fn);
  const int64_t nb_cap = (dims->prefix_cap + rswa::kBlock - 1) / rswa::kBlock;
  if (nb_cap > rswa::kMaxRouteBlocks)
    return fail(RSWA_ERR_UNSUPPORTED, "%s: %lld prefix blocks exceed the router's limit of %d", fn,
                (long long)nb_cap, rswa::kMaxRouteBlocks);
  if (nb_cap == 0) return fail(RSWA_ERR_INVALID, "%s: prefix_cap must be >= 1", fn);
  if (ws_bytes < 256) return fail(RSWA_ERR_INVALID, "%s: workspace must be at least 256 bytes", fn);
  cudaError_t e = rswa::launch_route(dims->batch, tokens, dims->prefix_cap, q_idx, kbar, prefix_len, idx_scale, topk,
                                     blk_idx, blk_logp, probs, tau, ws_status(workspace),
                                     static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, fn);
  return ok();
}

rswa_status srswa_route(const rswa_dims* dims, const float* q_idx, const float* kbar, const int32_t* prefix_len,
                        float idx_scale, int32_t topk, int32_t* blk_idx, float* blk_logp, float* probs, float* tau,
                        void* workspace, size_t ws_bytes, void* stream) {
  return route_common("srswa_route", dims, 1, q_idx, kbar, prefix_len, idx_scale, topk, blk_idx, blk_logp, probs,
                      tau, workspace, ws_bytes, stream);
}

rswa_status srswa_route_tokens(const rswa_dims* dims, int32_t T, const float* q_idx, const float* kbar,
                               const int32_t* prefix_len, float idx_scale, int32_t topk, int32_t* blk_idx,
                               float* blk_logp, void* workspace, size_t ws_bytes, void* stream) {
  return route_common("srswa_route_tokens", dims, T, q_idx, kbar, prefix_len, idx_scale, topk, blk_idx, blk_logp,
                      nullptr, nullptr, workspace, ws_bytes, stream);
}

size_t srswa_prefill_workspace_bytes(const rswa_dims* dims, int32_t T) {
  const char* fn = "srswa_prefill_workspace_bytes";
  if (check_dims(fn, dims, true) != RSWA_OK) return 0;
  if (T < 1) {
    fail(RSWA_ERR_INVALID, "%s: T must be >= 1 (got %d)", fn, T);
    return 0;
  }
  return 256 + rswa::srswa_prefill_scratch_bytes(dims->batch, dims->heads, T);
}

rswa_status srswa_prefill(const rswa_dims* dims, int32_t T, const void* q, const void* k_out, const void* v_out,
                          const void* pk, const void* pv, const int32_t* prefix_len, const int32_t* blk_idx,
                          const float* blk_logp, int32_t topk, const void* ring_k, const void* ring_v,
                          const int32_t* wp, const int32_t* fill, float scale, float* out, float* lse,
                          void* workspace, size_t ws_bytes, void* stream) {
  const char* fn = "srswa_prefill";
  const NvtxRange nvtx_range(fn);
  g_test_drop_tile = -1;  // the wait-timeout test hook covers the decode kernels only
  g_test_wait_ns = 0;
  rswa_status st = check_dims(fn, dims, true);
  if (st != RSWA_OK) return st;
  if (T < 1) return fail(RSWA_ERR_INVALID, "%s: T must be >= 1 (got %d)", fn, T);
  if (T > 8192) return fail(RSWA_ERR_UNSUPPORTED, "%s: chunks of more than 8192 queries (got %d)", fn, T);
  REQUIRE_PTR(q);
  REQUIRE_PTR(k_out);
  REQUIRE_PTR(v_out);
  if (dims->prefix_cap > 0) {
    REQUIRE_PTR(pk);
    REQUIRE_PTR(pv);
  }
  REQUIRE_PTR(out);
  REQUIRE_PTR(workspace);
  REQUIRE_PTR_OR_NULL(lse);
  if (prefix_len == nullptr) return fail(RSWA_ERR_INVALID, "%s: prefix_len must not be NULL", fn);
  if (blk_idx == nullptr || blk_logp == nullptr)
    return fail(RSWA_ERR_INVALID, "%s: blk_idx and blk_logp must not be NULL", fn);
  if (topk < 1 || topk > rswa::kMaxTopk) return fail(RSWA_ERR_INVALID, "%s: topk must be in [1, 32] (got %d)", fn, topk);
  if ((ring_k == nullptr) != (ring_v == nullptr))
    return fail(RSWA_ERR_INVALID, "%s: ring_k and ring_v must both be given or both be NULL", fn);
  const bool ring = ring_k != nullptr;
  if (ring) {
    REQUIRE_PTR(ring_k);
    REQUIRE_PTR(ring_v);
    if (wp == nullptr || fill == nullptr) return fail(RSWA_ERR_INVALID, "%s: a ring needs wp and fill", fn);
  }
  if (!(scale > 0.f) || !std::isfinite(scale)) return fail(RSWA_ERR_INVALID, "%s: scale must be finite and > 0", fn);
  const int64_t bh = (int64_t)dims->batch * dims->heads;
  const int64_t lim = ((int64_t)1 << 31) - 1;
  if (bh * T >= lim || bh * dims->prefix_cap >= lim || bh * dims->ring >= lim)
    return fail(RSWA_ERR_UNSUPPORTED, "%s: more than 2^31 rows in one operand", fn);
  const size_t need = 256 + rswa::srswa_prefill_scratch_bytes(dims->batch, dims->heads, T);
  if (ws_bytes < need)
    return fail(RSWA_ERR_INVALID, "%s: workspace of %zu bytes is smaller than the %zu required "
                "(srswa_prefill_workspace_bytes)", fn, ws_bytes, need);
  // workspace: [status 256 B][counts 256 B][group records][query lists][sorted routes][biases][lse of the band part]
  // [sort keys]
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const size_t bt = (size_t)dims->batch * T;
  int32_t* counts = reinterpret_cast<int32_t*>(ws + 256);
  int32_t* rec = reinterpret_cast<int32_t*>(ws + 512);
  int32_t* gq = reinterpret_cast<int32_t*>(ws + 512 + align256(bt * rswa::srswa_prefill_group_rec_ints() * 4));
  int32_t* gblk = reinterpret_cast<int32_t*>(reinterpret_cast<uint8_t*>(gq) + align256(bt * 4));
  float* gbias = reinterpret_cast<float*>(gblk + bt * rswa::kMaxTopk);
  float* lse_scratch = gbias + bt * rswa::kMaxTopk;
  uint64_t* keys = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(lse_scratch) +
                                               align256((size_t)dims->batch * dims->heads * T * 4));
  float* lse_use = lse != nullptr ? lse : lse_scratch;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // 1. group the chunk's queries by routed block set
  const bool routed = dims->prefix_cap > 0;  // with no prefix rows there is nothing to route to
  cudaError_t e = cudaSuccess;
  if (routed) {
    e = cudaMemsetAsync(counts, 0, 16, s);
    if (e != cudaSuccess) return cuda_fail(e, "srswa_prefill: clearing the group counters");
    e = rswa::launch_srswa_group(dims->batch, T, topk, dims->prefix_cap, prefix_len, blk_idx, blk_logp, rec, gq,
                                 gblk, gbias, counts, keys, ws_status(workspace), s);
    if (e != cudaSuccess) return cuda_fail(e, "srswa_prefill: grouping");
  }
  // 2. the band (and previous-chunk ring) part of every query: the dense tcgen05 prefill, prefix left out
  rswa::PrefillLaunch L;
  L.B = dims->batch;
  L.H = dims->heads;
  L.n = dims->ring;
  L.T = T;
  L.cap = dims->prefix_cap;
  L.q = q;
  L.k_out = k_out;
  L.v_out = v_out;
  L.pk = pk;
  L.pv = pv;
  L.prefix_len = prefix_len;
  L.ring_k = ring ? ring_k : nullptr;
  L.ring_v = ring ? ring_v : nullptr;
  L.wp = wp;
  L.fill = fill;
  L.scale = scale;
  L.out = out;
  L.lse = lse_use;
  L.write_ring = 0;
  L.ring_k_w = nullptr;
  L.ring_v_w = nullptr;
  L.wp_w = nullptr;
  L.fill_w = nullptr;
  L.status = ws_status(workspace);
  L.ignore_prefix = 1;
  e = rswa::launch_prefill(L, s);
  if (e != cudaSuccess) return cuda_fail(e, "srswa_prefill: band part");
  if (!routed) return ok();
  // 3. the routed blocks of every group, per head, merged into (out, lse)
  e = rswa::launch_srswa_routed(dims->batch, dims->heads, T, topk, dims->prefix_cap, prefix_len, q, pk, pv, rec, gq,
                                gbias, counts, scale, out, lse_use, ws_status(workspace), s);
  if (e != cudaSuccess) return cuda_fail(e, "srswa_prefill: routed part");
  return ok();
}

// ---------------------------------------------------------------------------
// rswa_decode_noalloc: rswa_decode for callers that cannot allocate device
// memory. Some callers cannot call cudaMalloc at all: code that runs inside an
// allocator-free serving loop, plugins handed raw pointers by a host engine
// that owns every allocation, or code paths that must not touch the caching
// allocator. For them the split-KV scratch (status word, per-(sequence, head)
// completion counters and partial results) lives in the file-scope device
// array below instead of a caller-provided workspace. Every GPU that loads
// this library holds the array until the process exits.
// ---------------------------------------------------------------------------
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;  // 4 MiB
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device. The array's
// name in host code is only a host-side stand-in, so the address is asked of
// the runtime once per device, with that device current.
rswa_status noalloc_scratch(const char* fn, uint8_t** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "rswa_decode_noalloc: cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(RSWA_ERR_UNSUPPORTED, "%s: device ordinal %d >= %d", fn, dev, kMaxDevices);
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "rswa_decode_noalloc: cudaGetSymbolAddress of the scratch array");
    g_noalloc_addr[dev] = p;
  }
  *out = static_cast<uint8_t*>(g_noalloc_addr[dev]);
  return RSWA_OK;
}

}  // namespace

rswa_status rswa_decode_noalloc(const rswa_dims* dims, const void* q, const void* pk, const void* pv,
                                const int32_t* prefix_len, const void* ring_k, const void* ring_v,
                                const int32_t* wp, const int32_t* fill, float scale, float* out, float* lse,
                                int32_t* status, void* stream) {
  const char* fn = "rswa_decode_noalloc";
  const NvtxRange nvtx_range(fn);
  rswa_status st = check_dims(fn, dims, true);
  if (st != RSWA_OK) return st;
  REQUIRE_PTR(q);
  REQUIRE_PTR(pk);
  REQUIRE_PTR(pv);
  REQUIRE_PTR(ring_k);
  REQUIRE_PTR(ring_v);
  REQUIRE_PTR(out);
  REQUIRE_PTR_OR_NULL(status);
  if (prefix_len == nullptr || wp == nullptr || fill == nullptr)
    return fail(RSWA_ERR_INVALID, "%s: prefix_len, wp and fill must not be NULL", fn);
  if (!(scale > 0.f) || !std::isfinite(scale)) return fail(RSWA_ERR_INVALID, "%s: scale must be finite and > 0", fn);
  const rswa::WorkspacePlan plan =
      rswa::plan_decode_workspace(dims->batch, dims->heads, rswa::decode_max_tiles_dense(dims->prefix_cap, dims->ring),
                                  rswa::device_sm_count(), kNoAllocScratchBytes);
  if (plan.bytes > kNoAllocScratchBytes)
    return fail(RSWA_ERR_UNSUPPORTED,
                "%s: these dims need %zu bytes of scratch, above the %zu-byte static scratch; use rswa_decode "
                "with a caller-provided workspace",
                fn, plan.bytes, kNoAllocScratchBytes);
  uint8_t* scratch = nullptr;
  st = noalloc_scratch(fn, &scratch);
  if (st != RSWA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // The array keeps the previous call's contents: zero the status word and the
  // completion counters (everything before the partials) before this call.
  cudaError_t e = cudaMemsetAsync(scratch, 0, plan.partials_off, s);
  if (e != cudaSuccess) return cuda_fail(e, "rswa_decode_noalloc: clearing the scratch counters");
  st = decode_common(fn, false, dims, q, bf16_prefix(pk, pv), kNoBand, kNoAppend, prefix_len, nullptr, nullptr, 0,
                     ring_k, ring_v, wp,
                     fill, scale, out, lse, scratch, kNoAllocScratchBytes, stream, kNoAllocScratchBytes);
  if (st != RSWA_OK) return st;
  if (status != nullptr) {
    e = cudaMemcpyAsync(status, scratch, sizeof(int32_t), cudaMemcpyDeviceToDevice, s);
    if (e != cudaSuccess) return cuda_fail(e, "rswa_decode_noalloc: copying the status word");
  }
  return ok();
}

}  // extern "C"
