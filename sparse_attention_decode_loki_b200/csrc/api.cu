// C ABI of the Loki library (declared in include/loki.h): argument checks,
// workspace carving and the launch sequence of each entry point. Every check
// runs on the host before anything is enqueued, so a rejected call launches
// nothing and touches no device memory.
#include <math.h>

#include <cstdarg>
#include <cstdio>
#include <string>

#include "../../include/loki.h"
#include "launch.h"

namespace {

thread_local std::string g_last_error;

loki_status fail(loki_status st, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return st;
}

loki_status cuda_fail(cudaError_t e, const char* where) {
    return fail(LOKI_ERR_CUDA, "%s: %s (%s)", where, cudaGetErrorName(e), cudaGetErrorString(e));
}

size_t align_up(size_t x, size_t a = 256) { return (x + a - 1) / a * a; }

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

constexpr int kMaxGroup = 8;
constexpr int64_t kMaxS = 0x7fffffff;

#define LOKI_REQUIRE(cond, st, ...) \
    do {                            \
        if (!(cond)) return fail(st, __VA_ARGS__); \
    } while (0)

loki_status check_dtype(loki_dtype dt) {
    LOKI_REQUIRE(dt == LOKI_DTYPE_F32 || dt == LOKI_DTYPE_BF16, LOKI_ERR_INVALID_ARG,
                 "dt must be LOKI_DTYPE_F32 or LOKI_DTYPE_BF16 (got %d)", (int)dt);
    return LOKI_OK;
}

loki_status check_heads(int B, int H_q, int H_kv, int D) {
    LOKI_REQUIRE(B >= 1 && B <= 65535, LOKI_ERR_INVALID_ARG, "B must be in [1, 65535] (got %d)", B);
    LOKI_REQUIRE(H_q >= 1 && H_kv >= 1, LOKI_ERR_INVALID_ARG, "H_q and H_kv must be >= 1");
    LOKI_REQUIRE(H_q % H_kv == 0, LOKI_ERR_INVALID_ARG, "H_q (%d) must be a multiple of H_kv (%d)",
                 H_q, H_kv);
    LOKI_REQUIRE(H_q / H_kv <= kMaxGroup, LOKI_ERR_UNSUPPORTED,
                 "H_q / H_kv = %d exceeds the supported group size %d", H_q / H_kv, kMaxGroup);
    LOKI_REQUIRE(D >= 1, LOKI_ERR_INVALID_ARG, "D must be >= 1");
    LOKI_REQUIRE(D == 128 || D == 96, LOKI_ERR_UNSUPPORTED,
                 "D = %d: head dimensions 128 and 96 are implemented", D);
    LOKI_REQUIRE((int64_t)B * H_q <= 0x7fffffff, LOKI_ERR_INVALID_ARG, "B * H_q too large");
    return LOKI_OK;
}

loki_status check_seq(int64_t S, int64_t S_max) {
    LOKI_REQUIRE(S >= 1, LOKI_ERR_INVALID_ARG, "S must be >= 1 (got %lld)", (long long)S);
    LOKI_REQUIRE(S <= S_max, LOKI_ERR_INVALID_ARG, "S (%lld) must be <= S_max (%lld)",
                 (long long)S, (long long)S_max);
    LOKI_REQUIRE(S <= kMaxS, LOKI_ERR_UNSUPPORTED, "S must be < 2^31 (int32 token indices)");
    return LOKI_OK;
}

loki_status check_plane(int d_lo, int D, loki_dtype dt) {
    const int e = dt == LOKI_DTYPE_F32 ? 4 : 2;
    LOKI_REQUIRE(d_lo >= 1 && d_lo <= D, LOKI_ERR_INVALID_ARG, "d_lo must be in [1, D] (got %d)",
                 d_lo);
    LOKI_REQUIRE((d_lo * e) % 16 == 0, LOKI_ERR_INVALID_ARG,
                 "d_lo * element size must be a multiple of 16 bytes (got d_lo = %d)", d_lo);
    return LOKI_OK;
}

#define LOKI_CHECK(expr)                    \
    do {                                    \
        loki_status st_ = (expr);           \
        if (st_ != LOKI_OK) return st_;     \
    } while (0)

#define LOKI_PTR(p, a)                                                                     \
    do {                                                                                   \
        LOKI_REQUIRE((p) != nullptr, LOKI_ERR_INVALID_ARG, "%s must not be NULL", #p);    \
        LOKI_REQUIRE(aligned((p), (a)), LOKI_ERR_INVALID_ARG, "%s must be %d-byte aligned", \
                     #p, (int)(a));                                                        \
    } while (0)

#define LOKI_CUDA(expr, where)                        \
    do {                                              \
        cudaError_t e_ = (expr);                      \
        if (e_ != cudaSuccess) return cuda_fail(e_, where); \
    } while (0)

loki::Dt to_dt(loki_dtype dt) { return dt == LOKI_DTYPE_F32 ? loki::kF32 : loki::kBF16; }

float resolve_scale(float scale, int D) {
    return (scale > 0.f && isfinite(scale)) ? scale : 1.0f / sqrtf((float)D);
}

// workspace pieces of the decode path
struct DecodeWs {
    size_t q_rot, scores, done, ml, acc, total;
};
DecodeWs decode_ws(int B, int H_q, int64_t S, int D, int64_t k) {
    const int64_t rows = (int64_t)B * H_q;
    const int64_t parts = loki::sparse_max_parts(rows, k);
    DecodeWs w;
    w.q_rot = 0;
    w.scores = align_up(w.q_rot + (size_t)rows * D * sizeof(float));
    w.done = align_up(w.scores + (size_t)rows * S * sizeof(float));
    w.ml = align_up(w.done + (size_t)rows * sizeof(int));
    w.acc = align_up(w.ml + (size_t)rows * parts * sizeof(float2));
    w.total = align_up(w.acc + (size_t)rows * parts * D * sizeof(float));
    return w;
}

// Paged decode: the work-split area of the paged scan, then a decode
// workspace for rows of S_cap = page_size * max_pages scores.
constexpr int kPagedMaxGrid = 1024;  // >= the scan grid (one CTA per SM)
struct PagedWs {
    size_t start, dec, total;
};
PagedWs paged_ws(int B, int H_q, int64_t S_cap, int D, int64_t k) {
    PagedWs w;
    w.start = 0;
    w.dec = align_up(loki::paged_start_bytes(B, kPagedMaxGrid));
    w.total = w.dec + decode_ws(B, H_q, S_cap, D, k).total;
    return w;
}

struct SparseWs {
    size_t done, ml, acc, total;
};
SparseWs sparse_ws(int B, int H_q, int64_t k, int D) {
    const int64_t rows = (int64_t)B * H_q;
    const int64_t parts = loki::sparse_max_parts(rows, k);
    SparseWs w;
    w.done = 0;
    w.ml = align_up((size_t)rows * sizeof(int));
    w.acc = align_up(w.ml + (size_t)rows * parts * sizeof(float2));
    w.total = align_up(w.acc + (size_t)rows * parts * D * sizeof(float));
    return w;
}

struct DenseWs {
    size_t ml, acc, total;
};
DenseWs dense_ws(int B, int H_q, int64_t S, int D) {
    // slots: units (B * H_kv) x parts x G = B * H_q x parts
    const int64_t slots = (int64_t)B * H_q * loki::dense_max_parts(S);
    DenseWs w;
    w.ml = 0;
    w.acc = align_up((size_t)slots * sizeof(float2));
    w.total = align_up(w.acc + (size_t)slots * D * sizeof(float));
    return w;
}

struct CalWs {
    size_t mean, cov, vec, total;
};
CalWs cal_ws(int H_kv, int D) {
    CalWs w;
    w.mean = 0;
    w.cov = align_up((size_t)H_kv * D * sizeof(double));
    w.vec = align_up(w.cov + (size_t)H_kv * D * D * sizeof(double));
    w.total = align_up(w.vec + (size_t)H_kv * D * D * sizeof(double));
    return w;
}

template <class T>
T* at(void* base, size_t off) {
    return reinterpret_cast<T*>(static_cast<char*>(base) + off);
}

}  // namespace

namespace loki {
void set_last_error(const char* msg) { g_last_error = msg; }
}  // namespace loki

extern "C" {

const char* loki_status_string(loki_status st) {
    switch (st) {
        case LOKI_OK: return "LOKI_OK";
        case LOKI_ERR_INVALID_ARG: return "LOKI_ERR_INVALID_ARG: invalid argument";
        case LOKI_ERR_UNSUPPORTED: return "LOKI_ERR_UNSUPPORTED: unsupported configuration";
        case LOKI_ERR_WORKSPACE_TOO_SMALL: return "LOKI_ERR_WORKSPACE_TOO_SMALL: workspace too small";
        case LOKI_ERR_CUDA: return "LOKI_ERR_CUDA: CUDA runtime error";
    }
    return "unknown loki_status";
}

const char* loki_last_error(void) { return g_last_error.c_str(); }

loki_status loki_device_error(int* code, int reset) {
    g_last_error.clear();
    LOKI_REQUIRE(code != nullptr, LOKI_ERR_INVALID_ARG, "code must not be NULL");
    int* w = loki::device_error_word();
    LOKI_REQUIRE(w != nullptr, LOKI_ERR_CUDA, "no usable current CUDA device");
    LOKI_CUDA(cudaMemcpy(code, w, sizeof(int), cudaMemcpyDeviceToHost), "loki_device_error");
    if (reset) LOKI_CUDA(cudaMemset(w, 0, sizeof(int)), "loki_device_error");
    return LOKI_OK;
}

// ---------------------------------------------------------------------------

size_t loki_calibrate_workspace_size(int64_t N, int H_kv, int D) {
    (void)N;
    if (H_kv < 1 || D < 1) return 0;
    return cal_ws(H_kv, D).total;
}

loki_status loki_calibrate_pca(const void* keys, loki_dtype dt, int64_t N, int H_kv, int D,
                               float* P, float* eigvals, void* ws, size_t ws_bytes,
                               void* stream) {
    g_last_error.clear();
    LOKI_CHECK(check_dtype(dt));
    LOKI_REQUIRE(N >= 2, LOKI_ERR_INVALID_ARG, "N must be >= 2 (got %lld)", (long long)N);
    LOKI_REQUIRE(H_kv >= 1 && H_kv <= 65535, LOKI_ERR_INVALID_ARG, "H_kv must be in [1, 65535]");
    LOKI_REQUIRE(D >= 16 && D <= 128 && D % 16 == 0, LOKI_ERR_UNSUPPORTED,
                 "calibration supports D in {16, 32, ..., 128} (got %d)", D);
    LOKI_PTR(keys, 16);
    LOKI_PTR(P, 16);
    if (eigvals) LOKI_PTR(eigvals, 4);
    LOKI_PTR(ws, 256);
    const CalWs w = cal_ws(H_kv, D);
    LOKI_REQUIRE(ws_bytes >= w.total, LOKI_ERR_WORKSPACE_TOO_SMALL,
                 "workspace %zu bytes < required %zu", ws_bytes, w.total);
    LOKI_CUDA(loki::launch_calibrate(to_dt(dt), keys, N, H_kv, D, P, eigvals, at<double>(ws, w.mean),
                                     at<double>(ws, w.cov), at<double>(ws, w.vec),
                                     static_cast<cudaStream_t>(stream)),
              "loki_calibrate_pca");
    return LOKI_OK;
}

loki_status loki_append_keys(const void* K_new, const void* V_new, const float* P,
                             void* Kt_cache, void* V_cache, int B, int H_kv, int T, int D,
                             int64_t S_max, int64_t pos, loki_dtype dt, void* stream) {
    g_last_error.clear();
    LOKI_CHECK(check_dtype(dt));
    LOKI_CHECK(check_heads(B, H_kv, H_kv, D));
    LOKI_REQUIRE(T >= 1, LOKI_ERR_INVALID_ARG, "T must be >= 1 (got %d)", T);
    LOKI_REQUIRE(pos >= 0 && S_max >= 1 && pos + T <= S_max, LOKI_ERR_INVALID_ARG,
                 "need 0 <= pos and pos + T <= S_max (pos %lld, T %d, S_max %lld)",
                 (long long)pos, T, (long long)S_max);
    LOKI_PTR(K_new, 16);
    LOKI_PTR(V_new, 16);
    LOKI_PTR(P, 16);
    LOKI_PTR(Kt_cache, 16);
    LOKI_PTR(V_cache, 16);
    LOKI_CUDA(loki::launch_append(to_dt(dt), K_new, V_new, P, Kt_cache, V_cache, nullptr, 0, B,
                                  H_kv, T, D, S_max, pos, static_cast<cudaStream_t>(stream)),
              "loki_append_keys");
    return LOKI_OK;
}

loki_status loki_append_keys_plane(const void* K_new, const void* V_new, const float* P,
                                   void* Kt_cache, void* V_cache, void* Kt_lo, int d_lo, int B,
                                   int H_kv, int T, int D, int64_t S_max, int64_t pos,
                                   loki_dtype dt, void* stream) {
    g_last_error.clear();
    LOKI_CHECK(check_dtype(dt));
    LOKI_CHECK(check_heads(B, H_kv, H_kv, D));
    LOKI_CHECK(check_plane(d_lo, D, dt));
    LOKI_REQUIRE(T >= 1, LOKI_ERR_INVALID_ARG, "T must be >= 1 (got %d)", T);
    LOKI_REQUIRE(pos >= 0 && S_max >= 1 && pos + T <= S_max, LOKI_ERR_INVALID_ARG,
                 "need 0 <= pos and pos + T <= S_max (pos %lld, T %d, S_max %lld)",
                 (long long)pos, T, (long long)S_max);
    LOKI_PTR(K_new, 16);
    LOKI_PTR(V_new, 16);
    LOKI_PTR(P, 16);
    LOKI_PTR(Kt_cache, 16);
    LOKI_PTR(V_cache, 16);
    LOKI_PTR(Kt_lo, 16);
    LOKI_CUDA(loki::launch_append(to_dt(dt), K_new, V_new, P, Kt_cache, V_cache, Kt_lo, d_lo, B,
                                  H_kv, T, D, S_max, pos, static_cast<cudaStream_t>(stream)),
              "loki_append_keys_plane");
    return LOKI_OK;
}

// ---------------------------------------------------------------------------

size_t loki_decode_workspace_size(int B, int H_q, int H_kv, int64_t S, int D, int d, int64_t k) {
    (void)H_kv;
    (void)d;
    if (B < 1 || H_q < 1 || S < 1 || D < 1 || k < 1) return 0;
    return decode_ws(B, H_q, S, D, k).total;
}

static loki_status check_decode_common(int B, int H_q, int H_kv, int64_t S, int64_t S_max, int D,
                                       loki_dtype dt) {
    LOKI_CHECK(check_dtype(dt));
    LOKI_CHECK(check_heads(B, H_q, H_kv, D));
    LOKI_CHECK(check_seq(S, S_max));
    return LOKI_OK;
}

// Selection and attention after the score scan (both programmatic dependents).
// d: the columns the scores cover, q_rot's own (the attention then adds the
// stored score and reads only the remaining key columns); 0 when the scores
// come from other queries or keys (the pre-rotary decode).
static loki_status decode_tail(const char* name, loki::Dt t, float* scores, float* q_rot,
                               int* done, void* ws, const DecodeWs& w, const void* Kt_cache,
                               const void* V_cache, int B, int H_q, int H_kv, int64_t S,
                               int64_t S_max, int D, int d, int64_t k, float scale, void* out,
                               int32_t* selected_idx, cudaStream_t s) {
    const int rows = B * H_q;
    if (loki::select_attend_fits(t, (int64_t)rows, S, D, k)) {
        // small decode: selection and attention in one persistent kernel
        LOKI_CUDA(loki::launch_select_attend(t, scores, q_rot, Kt_cache, V_cache, B, H_q, H_kv, S,
                                             S_max, k, resolve_scale(scale, D), out, selected_idx,
                                             s, true),
                  name);
        return LOKI_OK;
    }
    LOKI_CUDA(loki::launch_topk(scores, (int64_t)rows, S, k, selected_idx, s, true), name);
    // attention is a programmatic dependent of top-k too
    LOKI_CUDA(loki::launch_sparse_attention(t, q_rot, Kt_cache, V_cache, selected_idx, B, H_q, H_kv,
                                            S, S_max, D, k, resolve_scale(scale, D), out,
                                            at<float2>(ws, w.ml), at<float>(ws, w.acc), done, s,
                                            true, loki::PagedKV(), scores, d),
              name);
    return LOKI_OK;
}

// One decode step; with K_new (T new tokens per (batch, KV head)) the step
// first appends them at cache rows [S - T, S), rotated, in its first kernel.
static loki_status decode_impl(const char* name, const void* q, const void* Kt_cache,
                               const void* V_cache, const void* Kt_lo, int d_lo, const float* P,
                               int B, int H_q, int H_kv, int64_t S, int64_t S_max, int D, int d,
                               int64_t k, float scale, loki_dtype dt, void* out,
                               int32_t* selected_idx, void* ws, size_t ws_bytes, void* stream,
                               const void* K_new = nullptr, const void* V_new = nullptr,
                               int T = 0) {
    LOKI_CHECK(check_decode_common(B, H_q, H_kv, S, S_max, D, dt));
    LOKI_REQUIRE(d >= 1 && d <= D, LOKI_ERR_INVALID_ARG, "d must be in [1, D] (got %d)", d);
    LOKI_REQUIRE(k >= 1 && k <= S, LOKI_ERR_INVALID_ARG, "k must be in [1, S] (got %lld)",
                 (long long)k);
    LOKI_PTR(q, 16);
    LOKI_PTR(Kt_cache, 16);
    LOKI_PTR(V_cache, 16);
    LOKI_PTR(P, 16);
    LOKI_PTR(out, 16);
    LOKI_PTR(selected_idx, 4);
    LOKI_PTR(ws, 256);
    if (Kt_lo != nullptr) {
        LOKI_CHECK(check_plane(d_lo, D, dt));
        LOKI_PTR(Kt_lo, 16);
        LOKI_REQUIRE(d <= d_lo, LOKI_ERR_INVALID_ARG, "d (%d) must be <= d_lo (%d)", d, d_lo);
    }
    if (K_new != nullptr) {
        LOKI_PTR(K_new, 16);
        LOKI_PTR(V_new, 16);
        LOKI_REQUIRE(T >= 1 && T <= S, LOKI_ERR_INVALID_ARG,
                     "T must be in [1, S] new tokens (got %d)", T);
    }
    const DecodeWs w = decode_ws(B, H_q, S, D, k);
    LOKI_REQUIRE(ws_bytes >= w.total, LOKI_ERR_WORKSPACE_TOO_SMALL,
                 "workspace %zu bytes < required %zu", ws_bytes, w.total);
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    const loki::Dt t = to_dt(dt);
    float* q_rot = at<float>(ws, w.q_rot);
    float* scores = at<float>(ws, w.scores);
    int* done = at<int>(ws, w.done);
    const int rows = B * H_q;
    if (K_new != nullptr && Kt_lo != nullptr &&
        loki::decode_cluster_preferred(t, B, H_q, H_kv, S, D, d_lo, k)) {
        // Few units: the append's rotation, then the one-kernel cluster decode
        // (which rotates its own queries) as its programmatic dependent
        LOKI_CUDA(loki::launch_append(t, K_new, V_new, P, const_cast<void*>(Kt_cache),
                                      const_cast<void*>(V_cache), const_cast<void*>(Kt_lo), d_lo,
                                      B, H_kv, T, D, S_max, S - T, s),
                  name);
        LOKI_CUDA(loki::launch_decode_cluster(t, q, P, Kt_lo, Kt_cache, V_cache, B, H_q, H_kv, S,
                                              S_max, d_lo, d, k, resolve_scale(scale, D), out,
                                              selected_idx, s, true),
                  name);
        return LOKI_OK;
    }
    if (K_new != nullptr) {
        // Append and decode: the first kernel rotates the queries and the new
        // keys (writing their cache, plane and value rows) with at most one
        // CTA per SM; the score scan is its programmatic dependent, runs
        // beside it and streams every older row first, waiting for it only
        // before the new rows.
        const int64_t pos = S - T;
        LOKI_CUDA(loki::launch_rotate(t, q, K_new, V_new, P, q_rot, const_cast<void*>(Kt_cache),
                                      const_cast<void*>(V_cache), const_cast<void*>(Kt_lo), d_lo,
                                      B, H_q, H_kv, T, D, S_max, pos, s, done, rows, false,
                                      nullptr, nullptr, true),
                  name);
        if (Kt_lo != nullptr) {
            const bool fuse = loki::score_plane_fuses(t, H_q / H_kv, d_lo, D);
            LOKI_CUDA(loki::launch_score_plane(t, q_rot, Kt_lo, B, H_q, H_kv, S, S_max, D, d_lo, d,
                                               scores, s, true, fuse ? q : nullptr,
                                               fuse ? P : nullptr, pos),
                      name);
        } else {
            LOKI_CUDA(loki::launch_score_lowdim(t, q_rot, Kt_cache, B, H_q, H_kv, S, S_max, D, D,
                                                d, scores, s, true),
                      name);
        }
        return decode_tail(name, t, scores, q_rot, done, ws, w, Kt_cache, V_cache, B, H_q, H_kv,
                           S, S_max, D, d, k, scale, out, selected_idx, s);
    }
    // Few (batch, KV head) units over a low-dim key plane: one kernel does
    // the whole step, each unit split over a cluster of CTAs.
    if (Kt_lo != nullptr && loki::decode_cluster_preferred(t, B, H_q, H_kv, S, D, d_lo, k)) {
        LOKI_CUDA(loki::launch_decode_cluster(t, q, P, Kt_lo, Kt_cache, V_cache, B, H_q, H_kv, S,
                                              S_max, d_lo, d, k, resolve_scale(scale, D), out,
                                              selected_idx, s),
                  name);
        return LOKI_OK;
    }
    // Over a low-dim key plane: the TMA-staged score scan, which rotates the
    // queries' first d_lo columns itself and streams keys at once, with the
    // full query projection (which also zeroes the attention kernel's row
    // counters) launched beside it; over the row layout: the projection,
    // then the register-staged scan. Then selection and attention: one
    // persistent kernel for small decodes, else top-k followed by attention
    // with its row merge. The first kernel is ordered normally
    // after whatever precedes the call; the rest use programmatic dependent
    // launch.
    const bool fused = Kt_lo != nullptr && loki::score_plane_fuses(t, H_q / H_kv, d_lo, D);
    if (fused) {
        LOKI_CUDA(loki::launch_score_plane(t, q_rot, Kt_lo, B, H_q, H_kv, S, S_max, D, d_lo, d,
                                           scores, s, false, q, P),
                  name);
        LOKI_CUDA(loki::launch_project_query(t, q, P, B, H_q, H_kv, D, q_rot, s, done, rows, true),
                  name);
    } else {
        LOKI_CUDA(loki::launch_project_query(t, q, P, B, H_q, H_kv, D, q_rot, s, done, rows),
                  name);
        if (Kt_lo != nullptr)
            LOKI_CUDA(loki::launch_score_plane(t, q_rot, Kt_lo, B, H_q, H_kv, S, S_max, D, d_lo,
                                               d, scores, s, true),
                      name);
        else
            LOKI_CUDA(loki::launch_score_lowdim(t, q_rot, Kt_cache, B, H_q, H_kv, S, S_max, D, D,
                                                d, scores, s, true),
                      name);
    }
    return decode_tail(name, t, scores, q_rot, done, ws, w, Kt_cache, V_cache, B, H_q, H_kv, S,
                       S_max, D, d, k, scale, out, selected_idx, s);
}

loki_status loki_decode_attention(const void* q, const void* Kt_cache, const void* V_cache,
                                  const float* P, int B, int H_q, int H_kv, int64_t S,
                                  int64_t S_max, int D, int d, int64_t k, float scale,
                                  loki_dtype dt, void* out, int32_t* selected_idx, void* ws,
                                  size_t ws_bytes, void* stream) {
    return decode_impl("loki_decode_attention", q, Kt_cache, V_cache, nullptr, 0, P, B, H_q, H_kv,
                       S, S_max, D, d, k, scale, dt, out, selected_idx, ws, ws_bytes, stream);
}

loki_status loki_decode_attention_plane(const void* q, const void* Kt_cache, const void* V_cache,
                                        const void* Kt_lo, int d_lo, const float* P, int B,
                                        int H_q, int H_kv, int64_t S, int64_t S_max, int D, int d,
                                        int64_t k, float scale, loki_dtype dt, void* out,
                                        int32_t* selected_idx, void* ws, size_t ws_bytes,
                                        void* stream) {
    if (Kt_lo == nullptr) {
        g_last_error = "Kt_lo must not be NULL";
        return LOKI_ERR_INVALID_ARG;
    }
    return decode_impl("loki_decode_attention_plane", q, Kt_cache, V_cache, Kt_lo, d_lo, P, B,
                       H_q, H_kv, S, S_max, D, d, k, scale, dt, out, selected_idx, ws, ws_bytes,
                       stream);
}

loki_status loki_decode_step(const void* q, const void* K_new, const void* V_new, const float* P,
                             void* Kt_cache, void* V_cache, void* Kt_lo, int d_lo, int B, int H_q,
                             int H_kv, int T, int64_t pos, int64_t S_max, int D, int d, int64_t k,
                             float scale, loki_dtype dt, void* out, int32_t* selected_idx, void* ws,
                             size_t ws_bytes, void* stream) {
    if (K_new == nullptr || V_new == nullptr) {
        g_last_error = "K_new and V_new must not be NULL";
        return LOKI_ERR_INVALID_ARG;
    }
    if (pos < 0 || T < 1 || pos > kMaxS - T) {
        g_last_error = "need pos >= 0, T >= 1 and pos + T < 2^31";
        return LOKI_ERR_INVALID_ARG;
    }
    return decode_impl("loki_decode_step", q, Kt_cache, V_cache, Kt_lo, d_lo, P, B, H_q, H_kv,
                       pos + T, S_max, D, d, k, scale, dt, out, selected_idx, ws, ws_bytes, stream,
                       K_new, V_new, T);
}

static loki_status check_pages(int page_size, int max_pages, int64_t n_pages, int H_kv) {
    LOKI_REQUIRE(page_size >= 1 && max_pages >= 1 && n_pages >= 1, LOKI_ERR_INVALID_ARG,
                 "page_size, max_pages and n_pages must be >= 1");
    LOKI_REQUIRE((int64_t)page_size * max_pages <= kMaxS, LOKI_ERR_UNSUPPORTED,
                 "page_size * max_pages must be < 2^31 tokens");
    LOKI_REQUIRE(n_pages * H_kv * (int64_t)page_size <= kMaxS, LOKI_ERR_UNSUPPORTED,
                 "the page pool must hold fewer than 2^31 rows (n_pages * H_kv * page_size)");
    return LOKI_OK;
}

size_t loki_paged_decode_workspace_size(int B, int H_q, int H_kv, int page_size, int max_pages,
                                        int D, int d, int64_t k) {
    (void)H_kv;
    (void)d;
    if (B < 1 || H_q < 1 || page_size < 1 || max_pages < 1 || D < 1 || k < 1) return 0;
    return paged_ws(B, H_q, (int64_t)page_size * max_pages, D, k).total;
}

loki_status loki_decode_attention_paged(const void* q, const void* Kt_pages, const void* V_pages,
                                        const void* Kt_lo_pages, int d_lo, const float* P,
                                        const int32_t* block_table, const int32_t* seq_lens,
                                        int B, int H_q, int H_kv, int page_size, int max_pages,
                                        int64_t n_pages, int D, int d, int64_t k, float scale,
                                        loki_dtype dt, void* out, int32_t* selected_idx,
                                        void* ws, size_t ws_bytes, void* stream) {
    g_last_error.clear();
    LOKI_CHECK(check_dtype(dt));
    LOKI_CHECK(check_heads(B, H_q, H_kv, D));
    LOKI_CHECK(check_pages(page_size, max_pages, n_pages, H_kv));
    LOKI_CHECK(check_plane(d_lo, D, dt));
    const int64_t S_cap = (int64_t)page_size * max_pages;
    LOKI_REQUIRE(d >= 1 && d <= d_lo, LOKI_ERR_INVALID_ARG, "d must be in [1, d_lo] (got %d)", d);
    LOKI_REQUIRE(k >= 1 && k <= S_cap, LOKI_ERR_INVALID_ARG,
                 "k must be in [1, page_size * max_pages] (got %lld)", (long long)k);
    const loki::Dt t = to_dt(dt);
    LOKI_REQUIRE(loki::paged_scan_supported(t, H_q / H_kv, d_lo), LOKI_ERR_UNSUPPORTED,
                 "the paged scan takes plane rows of 16, 32, 64 or 128 bytes with "
                 "(H_q / H_kv) * d_lo <= 64 elements");
    LOKI_REQUIRE(S_cap <= 262144, LOKI_ERR_UNSUPPORTED,
                 "paged decode selects from at most 262144 tokens per sequence");
    LOKI_PTR(q, 16);
    LOKI_PTR(Kt_pages, 16);
    LOKI_PTR(V_pages, 16);
    LOKI_PTR(Kt_lo_pages, 16);
    LOKI_PTR(P, 16);
    LOKI_PTR(block_table, 4);
    LOKI_PTR(seq_lens, 4);
    LOKI_PTR(out, 16);
    LOKI_PTR(selected_idx, 4);
    LOKI_PTR(ws, 256);
    const PagedWs pw = paged_ws(B, H_q, S_cap, D, k);
    LOKI_REQUIRE(ws_bytes >= pw.total, LOKI_ERR_WORKSPACE_TOO_SMALL,
                 "workspace %zu bytes < required %zu", ws_bytes, pw.total);
    const int grid = loki::paged_scan_grid();
    LOKI_REQUIRE(grid >= 1 && grid <= kPagedMaxGrid, LOKI_ERR_CUDA, "no usable current CUDA device");
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    const char* name = "loki_decode_attention_paged";
    void* start_ws = at<char>(ws, pw.start);
    void* dws = at<char>(ws, pw.dec);
    const DecodeWs w = decode_ws(B, H_q, S_cap, D, k);
    float* q_rot = at<float>(dws, w.q_rot);
    float* scores = at<float>(dws, w.scores);
    int* done = at<int>(dws, w.done);
    const int rows = B * H_q;
    // the rotated queries (and zeroed row counters), the lengths' work split,
    // the paged scan, then top-k per row length and the paged gather
    LOKI_CUDA(loki::launch_project_query(t, q, P, B, H_q, H_kv, D, q_rot, s, done, rows), name);
    LOKI_CUDA(loki::launch_paged_prefix(seq_lens, B, H_kv, S_cap, start_ws, grid, s), name);
    LOKI_CUDA(loki::launch_score_paged(t, q_rot, Kt_lo_pages, d_lo, block_table, start_ws, B, H_q,
                                       H_kv, page_size, max_pages, n_pages, S_cap, d, D, scores,
                                       grid, s),
              name);
    const int* lens = loki::paged_lens(start_ws, B);
    LOKI_CUDA(loki::launch_topk(scores, (int64_t)rows, S_cap, k, selected_idx, s, true, lens, H_q),
              name);
    loki::PagedKV pg;
    pg.block_table = block_table;
    pg.page_size = page_size;
    pg.max_pages = max_pages;
    pg.n_pages = n_pages;
    pg.lens = lens;
    LOKI_CUDA(loki::launch_sparse_attention(t, q_rot, Kt_pages, V_pages, selected_idx, B, H_q, H_kv,
                                            S_cap, S_cap, D, k, resolve_scale(scale, D), out,
                                            at<float2>(dws, w.ml), at<float>(dws, w.acc), done, s,
                                            true, pg, scores, d),
              name);
    return LOKI_OK;
}

loki_status loki_append_keys_paged(const void* K_new, const void* V_new, const float* P,
                                   void* Kt_pages, void* V_pages, void* Kt_lo_pages, int d_lo,
                                   const int32_t* block_table, const int32_t* positions, int B,
                                   int H_kv, int T, int page_size, int max_pages, int64_t n_pages,
                                   int D, loki_dtype dt, void* stream) {
    g_last_error.clear();
    LOKI_CHECK(check_dtype(dt));
    LOKI_CHECK(check_heads(B, H_kv, H_kv, D));
    LOKI_CHECK(check_pages(page_size, max_pages, n_pages, H_kv));
    LOKI_REQUIRE(T >= 1, LOKI_ERR_INVALID_ARG, "T must be >= 1 (got %d)", T);
    LOKI_PTR(K_new, 16);
    LOKI_PTR(V_new, 16);
    LOKI_PTR(P, 16);
    LOKI_PTR(Kt_pages, 16);
    LOKI_PTR(V_pages, 16);
    LOKI_PTR(block_table, 4);
    LOKI_PTR(positions, 4);
    if (Kt_lo_pages != nullptr) {
        LOKI_CHECK(check_plane(d_lo, D, dt));
        LOKI_PTR(Kt_lo_pages, 16);
    }
    loki::PagedKV pg;
    pg.block_table = block_table;
    pg.page_size = page_size;
    pg.max_pages = max_pages;
    pg.n_pages = n_pages;
    LOKI_CUDA(loki::launch_rotate(to_dt(dt), nullptr, K_new, V_new, P, nullptr, Kt_pages, V_pages,
                                  Kt_lo_pages, Kt_lo_pages != nullptr ? d_lo : 0, B, H_kv, H_kv, T,
                                  D, 0, 0, static_cast<cudaStream_t>(stream), nullptr, 0, false,
                                  &pg, positions),
              "loki_append_keys_paged");
    return LOKI_OK;
}

loki_status loki_decode_attention_fused(const void* q, const void* Kt_cache, const void* V_cache,
                                        const void* Kt_lo, int d_lo, const float* P, int B,
                                        int H_q, int H_kv, int64_t S, int64_t S_max, int D, int d,
                                        int64_t k, float scale, loki_dtype dt, void* out,
                                        int32_t* selected_idx, void* stream) {
    g_last_error.clear();
    LOKI_CHECK(check_decode_common(B, H_q, H_kv, S, S_max, D, dt));
    LOKI_REQUIRE(d >= 1 && d <= D, LOKI_ERR_INVALID_ARG, "d must be in [1, D] (got %d)", d);
    LOKI_REQUIRE(k >= 1 && k <= S, LOKI_ERR_INVALID_ARG, "k must be in [1, S] (got %lld)",
                 (long long)k);
    LOKI_PTR(q, 16);
    LOKI_PTR(Kt_cache, 16);
    LOKI_PTR(V_cache, 16);
    LOKI_PTR(Kt_lo, 16);
    LOKI_PTR(P, 16);
    LOKI_PTR(out, 16);
    LOKI_PTR(selected_idx, 4);
    LOKI_CHECK(check_plane(d_lo, D, dt));
    LOKI_REQUIRE(d <= d_lo, LOKI_ERR_INVALID_ARG, "d (%d) must be <= d_lo (%d)", d, d_lo);
    const loki::Dt t = to_dt(dt);
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    // few (batch, KV head) units: each unit split over a cluster of CTAs
    if (loki::decode_cluster_fits(t, B, H_q, H_kv, S, D, d_lo, k)) {
        LOKI_CUDA(loki::launch_decode_cluster(t, q, P, Kt_lo, Kt_cache, V_cache, B, H_q, H_kv, S,
                                              S_max, d_lo, d, k, resolve_scale(scale, D), out,
                                              selected_idx, s),
                  "loki_decode_attention_fused");
        return LOKI_OK;
    }
    LOKI_REQUIRE(loki::decode_fused_fits(t, H_q, H_kv, S, D, d_lo, k), LOKI_ERR_UNSUPPORTED,
                 "the fused decode kernel takes H_q / H_kv in {1, 2, 4, 8}, S <= 8192, plane "
                 "rows of 16, 32, 64 or 128 bytes, and keys that fit in shared memory");
    LOKI_CUDA(loki::launch_decode_fused(t, q, P, Kt_lo, Kt_cache, V_cache, B, H_q, H_kv, S, S_max,
                                        d_lo, d, k, resolve_scale(scale, D), out, selected_idx, s),
              "loki_decode_attention_fused");
    return LOKI_OK;
}

loki_status loki_project_query(const void* q, const float* P, int B, int H_q, int H_kv, int D,
                               loki_dtype dt, float* q_rot, void* stream) {
    g_last_error.clear();
    LOKI_CHECK(check_dtype(dt));
    LOKI_CHECK(check_heads(B, H_q, H_kv, D));
    LOKI_PTR(q, 16);
    LOKI_PTR(P, 16);
    LOKI_PTR(q_rot, 16);
    LOKI_CUDA(loki::launch_project_query(to_dt(dt), q, P, B, H_q, H_kv, D, q_rot,
                                         static_cast<cudaStream_t>(stream)),
              "project_query");
    return LOKI_OK;
}

loki_status loki_score_lowdim(const float* q_rot, const void* Kt_cache, int B, int H_q, int H_kv,
                              int64_t S, int64_t S_max, int D, int d, loki_dtype dt,
                              float* scores, void* stream) {
    g_last_error.clear();
    LOKI_CHECK(check_dtype(dt));
    // Kt_cache rows hold D elements: the rotated cache of 128- or 96-wide
    // heads (D = 128 or 96, and q_rot rows hold D), or a low-dimensional key
    // plane of 128-wide heads (any other D = d_lo; q_rot rows hold 128).
    const int Dq = (D == 96 || D == 128) ? D : 128;
    LOKI_CHECK(check_heads(B, H_q, H_kv, Dq));
    LOKI_CHECK(check_seq(S, S_max));
    LOKI_CHECK(check_plane(D, 128, dt));
    LOKI_REQUIRE(d >= 1 && d <= D, LOKI_ERR_INVALID_ARG, "d must be in [1, D] (got %d)", d);
    LOKI_PTR(q_rot, 16);
    LOKI_PTR(Kt_cache, 16);
    LOKI_PTR(scores, 4);
    // a plane (row width < 128) goes through the same TMA-staged scan as the
    // decode step; the rotated cache through the register-staged scan
    if (D < Dq)
        LOKI_CUDA(loki::launch_score_plane(to_dt(dt), q_rot, Kt_cache, B, H_q, H_kv, S, S_max, Dq,
                                           D, d, scores, static_cast<cudaStream_t>(stream), false),
                  "loki_score_lowdim");
    else
        LOKI_CUDA(loki::launch_score_lowdim(to_dt(dt), q_rot, Kt_cache, B, H_q, H_kv, S, S_max, Dq,
                                            D, d, scores, static_cast<cudaStream_t>(stream),
                                            false),
                  "loki_score_lowdim");
    return LOKI_OK;
}

size_t loki_topk_workspace_size(int64_t rows, int64_t S, int64_t k) {
    (void)rows;
    (void)S;
    (void)k;
    return 0;
}

loki_status loki_topk(const float* scores, int64_t rows, int64_t S, int64_t k,
                      int32_t* selected_idx, void* ws, size_t ws_bytes, void* stream) {
    g_last_error.clear();
    (void)ws;
    (void)ws_bytes;
    LOKI_REQUIRE(rows >= 1 && rows <= 0x7fffffff, LOKI_ERR_INVALID_ARG,
                 "rows must be in [1, 2^31) (got %lld)", (long long)rows);
    LOKI_REQUIRE(S >= 1 && S <= kMaxS, LOKI_ERR_INVALID_ARG, "S must be in [1, 2^31)");
    LOKI_REQUIRE(k >= 1 && k <= S, LOKI_ERR_INVALID_ARG, "k must be in [1, S] (got %lld)",
                 (long long)k);
    LOKI_PTR(scores, 4);
    LOKI_PTR(selected_idx, 4);
    LOKI_CUDA(loki::launch_topk(scores, rows, S, k, selected_idx, static_cast<cudaStream_t>(stream),
                                false),
              "topk");
    return LOKI_OK;
}

size_t loki_sparse_attention_workspace_size(int B, int H_q, int64_t k, int D) {
    if (B < 1 || H_q < 1 || k < 1 || D < 1) return 0;
    return sparse_ws(B, H_q, k, D).total;
}

loki_status loki_sparse_attention(const float* q_rot, const void* Kt_cache, const void* V_cache,
                                  const int32_t* selected_idx, int B, int H_q, int H_kv,
                                  int64_t S, int64_t S_max, int D, int64_t k, float scale,
                                  loki_dtype dt, void* out, void* ws, size_t ws_bytes,
                                  void* stream) {
    g_last_error.clear();
    LOKI_CHECK(check_decode_common(B, H_q, H_kv, S, S_max, D, dt));
    LOKI_REQUIRE(k >= 1 && k <= kMaxS, LOKI_ERR_INVALID_ARG, "k must be in [1, 2^31)");
    LOKI_PTR(q_rot, 16);
    LOKI_PTR(Kt_cache, 16);
    LOKI_PTR(V_cache, 16);
    LOKI_PTR(selected_idx, 4);
    LOKI_PTR(out, 16);
    LOKI_PTR(ws, 256);
    const SparseWs w = sparse_ws(B, H_q, k, D);
    LOKI_REQUIRE(ws_bytes >= w.total, LOKI_ERR_WORKSPACE_TOO_SMALL,
                 "workspace %zu bytes < required %zu", ws_bytes, w.total);
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    LOKI_CUDA(cudaMemsetAsync(at<int>(ws, w.done), 0, (size_t)B * H_q * sizeof(int), s),
              "sparse_attention");
    LOKI_CUDA(loki::launch_sparse_attention(to_dt(dt), q_rot, Kt_cache, V_cache, selected_idx, B,
                                            H_q, H_kv, S, S_max, D, k, resolve_scale(scale, D), out,
                                            at<float2>(ws, w.ml), at<float>(ws, w.acc),
                                            at<int>(ws, w.done), s, false),
              "sparse_attention");
    return LOKI_OK;
}

// ---------------------------------------------------------------------------

size_t loki_decode_prerotary_workspace_size(int B, int H_q, int H_kv, int64_t S, int D, int d,
                                            int64_t k) {
    (void)H_kv;
    (void)d;
    if (B < 1 || H_q < 1 || S < 1 || D < 1 || k < 1) return 0;
    return align_up((size_t)B * H_q * D * sizeof(float)) + decode_ws(B, H_q, S, D, k).total;
}

loki_status loki_decode_attention_prerotary(const void* q_pre, const void* q_post,
                                            const void* K_cache, const void* V_cache,
                                            const void* Kt_lo, int d_lo, const float* P, int B,
                                            int H_q, int H_kv, int64_t S, int64_t S_max, int D,
                                            int d, int64_t k, float scale, loki_dtype dt,
                                            void* out, int32_t* selected_idx, void* ws,
                                            size_t ws_bytes, void* stream) {
    g_last_error.clear();
    const char* name = "loki_decode_attention_prerotary";
    LOKI_CHECK(check_decode_common(B, H_q, H_kv, S, S_max, D, dt));
    LOKI_CHECK(check_plane(d_lo, D, dt));
    LOKI_REQUIRE(d >= 1 && d <= d_lo, LOKI_ERR_INVALID_ARG, "d must be in [1, d_lo] (got %d)", d);
    LOKI_REQUIRE(k >= 1 && k <= S, LOKI_ERR_INVALID_ARG, "k must be in [1, S] (got %lld)",
                 (long long)k);
    LOKI_PTR(q_pre, 16);
    LOKI_PTR(q_post, 16);
    LOKI_PTR(K_cache, 16);
    LOKI_PTR(V_cache, 16);
    LOKI_PTR(Kt_lo, 16);
    LOKI_PTR(P, 16);
    LOKI_PTR(out, 16);
    LOKI_PTR(selected_idx, 4);
    LOKI_PTR(ws, 256);
    const size_t qbytes = align_up((size_t)B * H_q * D * sizeof(float));
    const DecodeWs w = decode_ws(B, H_q, S, D, k);
    LOKI_REQUIRE(ws_bytes >= qbytes + w.total, LOKI_ERR_WORKSPACE_TOO_SMALL,
                 "workspace %zu bytes < required %zu", ws_bytes, qbytes + w.total);
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    const loki::Dt t = to_dt(dt);
    float* q_sc = at<float>(ws, 0);  // q~ = q_pre P, for the scores
    void* dws = at<char>(ws, qbytes);
    float* q_att = at<float>(dws, w.q_rot);  // q_post in fp32, for the attention
    float* scores = at<float>(dws, w.scores);
    int* done = at<int>(dws, w.done);
    const int rows = B * H_q;
    // the scan of the pre-rotary plane (rotating q_pre itself where it can);
    // q_post is widened to fp32 by the identity rotation
    if (loki::score_plane_fuses(t, H_q / H_kv, d_lo, D)) {
        LOKI_CUDA(loki::launch_score_plane(t, q_sc, Kt_lo, B, H_q, H_kv, S, S_max, D, d_lo, d,
                                           scores, s, false, q_pre, P),
                  name);
        LOKI_CUDA(loki::launch_project_query(t, q_post, nullptr, B, H_q, H_kv, D, q_att, s, done,
                                             rows, true),
                  name);
    } else {
        LOKI_CUDA(loki::launch_project_query(t, q_pre, P, B, H_q, H_kv, D, q_sc, s), name);
        LOKI_CUDA(loki::launch_project_query(t, q_post, nullptr, B, H_q, H_kv, D, q_att, s, done,
                                             rows),
                  name);
        LOKI_CUDA(loki::launch_score_plane(t, q_sc, Kt_lo, B, H_q, H_kv, S, S_max, D, d_lo, d,
                                           scores, s, true),
                  name);
    }
    // (the scores come from the pre-rotary queries and keys: no reuse)
    return decode_tail(name, t, scores, q_att, done, dws, w, K_cache, V_cache, B, H_q, H_kv, S,
                       S_max, D, 0, k, scale, out, selected_idx, s);
}

loki_status loki_append_keys_prerotary(const void* K_new_pre, const void* K_new_post,
                                       const void* V_new, const float* P, void* K_cache,
                                       void* V_cache, void* Kt_lo, int d_lo, int B, int H_kv,
                                       int T, int D, int64_t S_max, int64_t pos, loki_dtype dt,
                                       void* stream) {
    g_last_error.clear();
    LOKI_CHECK(check_dtype(dt));
    LOKI_CHECK(check_heads(B, H_kv, H_kv, D));
    LOKI_CHECK(check_plane(d_lo, D, dt));
    LOKI_REQUIRE(T >= 1, LOKI_ERR_INVALID_ARG, "T must be >= 1 (got %d)", T);
    LOKI_REQUIRE(pos >= 0 && S_max >= 1 && pos + T <= S_max, LOKI_ERR_INVALID_ARG,
                 "need 0 <= pos and pos + T <= S_max (pos %lld, T %d, S_max %lld)",
                 (long long)pos, T, (long long)S_max);
    LOKI_PTR(K_new_pre, 16);
    LOKI_PTR(K_new_post, 16);
    LOKI_PTR(V_new, 16);
    LOKI_PTR(P, 16);
    LOKI_PTR(K_cache, 16);
    LOKI_PTR(V_cache, 16);
    LOKI_PTR(Kt_lo, 16);
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    const loki::Dt t = to_dt(dt);
    const char* name = "loki_append_keys_prerotary";
    // the rotated pre-rotary keys go to the plane only; the post-rotary keys
    // (identity rotation) and the values to the caches
    LOKI_CUDA(loki::launch_rotate(t, nullptr, K_new_pre, nullptr, P, nullptr, nullptr, nullptr,
                                  Kt_lo, d_lo, B, H_kv, H_kv, T, D, S_max, pos, s, nullptr, 0,
                                  false),
              name);
    LOKI_CUDA(loki::launch_rotate(t, nullptr, K_new_post, V_new, nullptr, nullptr, K_cache,
                                  V_cache, nullptr, 0, B, H_kv, H_kv, T, D, S_max, pos, s, nullptr,
                                  0, false),
              name);
    return LOKI_OK;
}

size_t loki_pca_attention_workspace_size(int B, int H_q, int H_kv, int64_t S, int D) {
    (void)H_kv;
    if (B < 1 || H_q < 1 || S < 1 || D < 1) return 0;
    return align_up((size_t)B * H_q * D * sizeof(float)) + dense_ws(B, H_q, S, D).total;
}

loki_status loki_pca_attention(const void* q, const void* Kt_lo, int d_lo, const void* V_cache,
                               const float* P, int B, int H_q, int H_kv, int64_t S,
                               int64_t S_max, int D, int d, float scale, loki_dtype dt, void* out,
                               void* ws, size_t ws_bytes, void* stream) {
    g_last_error.clear();
    LOKI_CHECK(check_decode_common(B, H_q, H_kv, S, S_max, D, dt));
    LOKI_CHECK(check_plane(d_lo, D, dt));
    LOKI_REQUIRE(d >= 1 && d <= d_lo, LOKI_ERR_INVALID_ARG, "d must be in [1, d_lo] (got %d)", d);
    const loki::Dt t = to_dt(dt);
    LOKI_REQUIRE(loki::pca_attention_supported(t, d_lo), LOKI_ERR_UNSUPPORTED,
                 "PCAAttn takes plane rows of 16, 32, 64 or 128 bytes");
    LOKI_PTR(q, 16);
    LOKI_PTR(Kt_lo, 16);
    LOKI_PTR(V_cache, 16);
    LOKI_PTR(P, 16);
    LOKI_PTR(out, 16);
    LOKI_PTR(ws, 256);
    const size_t qbytes = align_up((size_t)B * H_q * D * sizeof(float));
    const DenseWs w = dense_ws(B, H_q, S, D);
    LOKI_REQUIRE(ws_bytes >= qbytes + w.total, LOKI_ERR_WORKSPACE_TOO_SMALL,
                 "workspace %zu bytes < required %zu", ws_bytes, qbytes + w.total);
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    float* q_rot = at<float>(ws, 0);
    void* dws = at<char>(ws, qbytes);
    LOKI_CUDA(loki::launch_project_query(t, q, P, B, H_q, H_kv, D, q_rot, s), "loki_pca_attention");
    LOKI_CUDA(loki::launch_pca_attention(t, q_rot, Kt_lo, d_lo, d, V_cache, B, H_q, H_kv, S, S_max,
                                         D, resolve_scale(scale, D), out, at<float2>(dws, w.ml),
                                         at<float>(dws, w.acc), s),
              "loki_pca_attention");
    return LOKI_OK;
}

size_t dense_decode_workspace_size(int B, int H_q, int H_kv, int64_t S, int D) {
    (void)H_kv;
    if (B < 1 || H_q < 1 || S < 1 || D < 1) return 0;
    return dense_ws(B, H_q, S, D).total;
}

loki_status dense_decode_attention(const void* q, const void* K_cache, const void* V_cache,
                                   int B, int H_q, int H_kv, int64_t S, int64_t S_max, int D,
                                   float scale, loki_dtype dt, void* out, void* ws,
                                   size_t ws_bytes, void* stream) {
    g_last_error.clear();
    LOKI_CHECK(check_decode_common(B, H_q, H_kv, S, S_max, D, dt));
    LOKI_PTR(q, 16);
    LOKI_PTR(K_cache, 16);
    LOKI_PTR(V_cache, 16);
    LOKI_PTR(out, 16);
    LOKI_PTR(ws, 256);
    const DenseWs w = dense_ws(B, H_q, S, D);
    LOKI_REQUIRE(ws_bytes >= w.total, LOKI_ERR_WORKSPACE_TOO_SMALL,
                 "workspace %zu bytes < required %zu", ws_bytes, w.total);
    LOKI_CUDA(loki::launch_dense(to_dt(dt), q, K_cache, V_cache, B, H_q, H_kv, S, S_max, D,
                                 resolve_scale(scale, D), out, at<float2>(ws, w.ml),
                                 at<float>(ws, w.acc), static_cast<cudaStream_t>(stream)),
              "dense_decode_attention");
    return LOKI_OK;
}

}  // extern "C"
