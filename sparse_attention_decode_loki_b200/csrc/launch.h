// Internal host-side launchers, one per kernel family. The C ABI (api.cu)
// validates arguments, carves workspaces and calls these; each returns the
// CUDA error of its launches.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace loki {

enum Dt : int { kF32 = 0, kBF16 = 1 };

// number of SMs and opt-in shared memory of the current device (cached)
struct DevInfo {
    int device;
    int sm_count;
    int smem_optin;
};
cudaError_t dev_info(DevInfo* out);

// resident CTAs per SM of `func` at `threads` threads and `smem` dynamic bytes (cached)
int occupancy(const void* func, int threads, size_t smem);

// device address of this device's kernel error word (cached; null on failure)
int* device_error_word();

// sets the text loki_last_error() returns on the calling thread
void set_last_error(const char* msg);

// ---- decode steps --------------------------------------------------------
// also zeroes done[0, n_done) when done is not null. With pdl it is launched
// as a programmatic dependent of the preceding kernel (the score scan that
// rotates its own queries) and runs beside it; it then completes only after
// that kernel does.
cudaError_t launch_project_query(Dt dt, const void* q, const float* P, int B, int H_q, int H_kv,
                                 int D, float* q_rot, cudaStream_t s, int* done = nullptr,
                                 int n_done = 0, bool pdl = false);

// `row` is the row length (and stride) of the key buffer scanned: D for the
// rotated cache, d_lo for a low-dimensional key plane.
cudaError_t launch_score_lowdim(Dt dt, const float* q_rot, const void* Kt, int B, int H_q,
                                int H_kv, int64_t S, int64_t S_max, int D, int row, int d,
                                float* scores, cudaStream_t s, bool pdl);

// Whether launch_score_plane can rotate the queries itself for this shape.
bool score_plane_fuses(Dt dt, int G, int d_lo, int D);

// TMA-staged scan of a low-dim key plane Klo [B, H_kv, S_max, d_lo]. With pdl
// it may start while the projection that writes q_rot is still running: it
// streams keys first and its consumers wait for q_rot. Given the raw queries
// q and the bases P (head dim 128; score_plane_fuses) the consumers rotate the
// query themselves, and the scan is launched without pdl whatever pdl says.
// wait_row < S: rows [wait_row, S) of every unit are written by the preceding
// kernel; the scan (launched as its programmatic dependent) streams the other
// rows at once and waits for it before reading those.
cudaError_t launch_score_plane(Dt dt, const float* q_rot, const void* Klo, int B, int H_q,
                               int H_kv, int64_t S, int64_t S_max, int D, int d_lo, int d,
                               float* scores, cudaStream_t s, bool pdl, const void* q = nullptr,
                               const float* P = nullptr, int64_t wait_row = INT64_MAX);

// With lens, row r holds min(lens[r / H_q], S) valid keys (at stride S) and
// selects min(k, that) of them, padding its k outputs with -1.
cudaError_t launch_topk(const float* scores, int64_t rows, int64_t S, int64_t k, int32_t* idx,
                        cudaStream_t s, bool pdl, const int* lens = nullptr, int H_q = 1);

// Whether the fused one-CTA-per-unit decode kernel can run this decode over a
// low-dim key plane: head dim 128; G in {1, 2, 4, 8}; S within the block
// top-k; plane rows of 1, 2, 4 or 8 16-byte chunks; the unit's keys and
// selection fit in shared memory.
bool decode_fused_fits(Dt dt, int H_q, int H_kv, int64_t S, int D, int d_lo, int64_t k);
// The whole decode step in one kernel: rotation, score scan over the plane,
// top-k and sparse attention, per (batch, KV head) unit; writes out and sel.
// The same step with each (batch, KV head) unit split over a cluster of 2-8
// CTAs (top-k through distributed shared memory), for decodes with few
// units: fits when D = 128, G in {1, 2, 4, 8}, plane rows of 16-128 bytes,
// S <= 8192, B * H_kv * 2 <= 2 * SMs and the keys fit in shared memory.
bool decode_cluster_fits(Dt dt, int B, int H_q, int H_kv, int64_t S, int D, int d_lo, int64_t k);
// Whether a plane decode takes it on its own: when it fits and there are at
// least 16 units (measured: faster than the four-kernel pipeline from 32
// units at S = 4096 and 40 units at S = 2048; slower for a single unit).
bool decode_cluster_preferred(Dt dt, int B, int H_q, int H_kv, int64_t S, int D, int d_lo,
                              int64_t k);
cudaError_t launch_decode_cluster(Dt dt, const void* q, const float* P, const void* Klo,
                                  const void* Kt, const void* V, int B, int H_q, int H_kv,
                                  int64_t S, int64_t S_max, int d_lo, int d, int64_t k,
                                  float scale, void* out, int32_t* sel, cudaStream_t s,
                                  bool pdl = false);
cudaError_t launch_decode_fused(Dt dt, const void* q, const float* P, const void* Klo,
                                const void* Kt, const void* V, int B, int H_q, int H_kv, int64_t S,
                                int64_t S_max, int d_lo, int d, int64_t k, float scale, void* out,
                                int32_t* sel, cudaStream_t s);

// Whether the decode takes the one-kernel selection + attention: small
// decodes (rows * k <= 8192, rows of at most 8192 keys, head dim 128).
bool select_attend_fits(Dt dt, int64_t rows, int64_t S, int D, int64_t k);
// Top-k of every (batch, query head) row of `scores` [B * H_q, S] and exact
// attention over the selected tokens, in one kernel: writes sel [B * H_q, k]
// and out [B * H_q, 128]. q_rot is q~ [B * H_q, 128] fp32.
cudaError_t launch_select_attend(Dt dt, const float* scores, const float* q_rot, const void* Kt,
                                 const void* V, int B, int H_q, int H_kv, int64_t S,
                                 int64_t S_max, int64_t k, float scale, void* out, int32_t* sel,
                                 cudaStream_t s, bool pdl);

// partial slots per (batch, query head) row of the sparse attention split
int64_t sparse_max_parts(int64_t rows, int64_t k);
// done[B*H_q] must be zero on entry (per-row completion counters; the last
// warp of a row merges its partials into out and leaves the counter at zero).
// Paged caches (block_table not null): Kt and V are page pools [n_pages, H_kv,
// page_size, D]; sequence b's token j is row j % page_size of page
// block_table[b * max_pages + j / page_size]. With lens, tokens at or beyond
// lens[b] (and pages outside the pool) are skipped.
struct PagedKV {
    const int* block_table = nullptr;
    int page_size = 0;
    int max_pages = 0;
    int64_t n_pages = 0;
    const int* lens = nullptr;
};
// sc_lo (optional): the decode's low-dim scores [rows, S] over the first d_sc
// columns (q~[:d_sc] . K~[:d_sc], as the score scan wrote them); the gather
// then reads only the remaining columns of each key row and adds the score.
cudaError_t launch_sparse_attention(Dt dt, const float* q_rot, const void* Kt, const void* V,
                                    const int32_t* idx, int B, int H_q, int H_kv, int64_t S,
                                    int64_t S_max, int D, int64_t k, float scale, void* out,
                                    float2* part_ml, float* part_acc, int* done, cudaStream_t s,
                                    bool pdl, const PagedKV& pg = PagedKV(),
                                    const float* sc_lo = nullptr, int d_sc = 0);

// ---- paged key plane -------------------------------------------------------
// One CTA per SM; the prefix kernel turns seq_lens into this grid's work split.
int paged_scan_grid();
// Bytes of the work-split area (lengths, row offsets, per-CTA starts).
size_t paged_start_bytes(int B, int grid);
bool paged_scan_supported(Dt dt, int G, int d_lo);
cudaError_t launch_paged_prefix(const int* seq_lens, int B, int H_kv, int64_t S_cap, void* start_ws,
                                int grid, cudaStream_t s);
// the clamped per-sequence lengths inside the work-split area
const int* paged_lens(const void* start_ws, int B);
cudaError_t launch_score_paged(Dt dt, const float* q_rot, const void* Klo_pages, int d_lo,
                               const int* block_table, const void* start_ws, int B, int H_q,
                               int H_kv, int page_size, int max_pages, int64_t n_pages,
                               int64_t S_cap, int d, int D, float* scores, int grid,
                               cudaStream_t s);

// split-S partial slots per (batch, KV head) unit
int64_t dense_max_parts(int64_t S);
cudaError_t launch_dense(Dt dt, const void* q, const void* K, const void* V, int B, int H_q,
                         int H_kv, int64_t S, int64_t S_max, int D, float scale, void* out,
                         float2* part_ml, float* part_acc, cudaStream_t s);

// Rotation into the KV heads' PCA bases, in one kernel: the G query rows of
// every (batch, KV head) into q_rot (q may be null), and T new keys per
// (batch, KV head) into cache rows [pos, pos + T) of Kt_cache (and of the plane
// Kt_lo when not null) with their values copied to V_cache (K_new may be
// null). Also zeroes done[0, n_done). With pdl it is a programmatic dependent
// of the preceding kernel that completes only after it (see the score scan).
// Paged (pg not null): the new keys of sequence b go to logical tokens
// positions[b] + t of its pages (rows whose page is missing are skipped and
// flag the device error word).
cudaError_t launch_rotate(Dt dt, const void* q, const void* K_new, const void* V_new,
                          const float* P, float* q_rot, void* Kt_cache, void* V_cache, void* Kt_lo,
                          int d_lo, int B, int H_q, int H_kv, int T, int D, int64_t S_max,
                          int64_t pos, cudaStream_t s, int* done, int n_done, bool pdl,
                          const PagedKV* pg = nullptr, const int* positions = nullptr,
                          bool one_per_sm = false);

// PCAAttn: softmax over the low-dimensional scores s_j = q~[:d] . K~_j[:d] of
// all S tokens (keys from the plane Klo [B, H_kv, S_max, d_lo]), out = sum p_j
// V_j. A programmatic dependent of the projection that writes q_rot.
bool pca_attention_supported(Dt dt, int d_lo);
cudaError_t launch_pca_attention(Dt dt, const float* q_rot, const void* Klo, int d_lo, int d,
                                 const void* V, int B, int H_q, int H_kv, int64_t S, int64_t S_max,
                                 int D, float scale, void* out, float2* part_ml, float* part_acc,
                                 cudaStream_t s);

// ---- supporting subsystems -----------------------------------------------
// Kt_lo (may be null): [B, H_kv, S_max, d_lo] plane that also receives the
// first d_lo rotated columns of each appended key.
cudaError_t launch_append(Dt dt, const void* K_new, const void* V_new, const float* P,
                          void* Kt_cache, void* V_cache, void* Kt_lo, int d_lo, int B, int H_kv,
                          int T, int D, int64_t S_max, int64_t pos, cudaStream_t s);

cudaError_t launch_calibrate(Dt dt, const void* keys, int64_t N, int H_kv, int D, float* P,
                             float* eigvals, double* ws_mean, double* ws_cov, double* ws_vec,
                             cudaStream_t s);

}  // namespace loki
