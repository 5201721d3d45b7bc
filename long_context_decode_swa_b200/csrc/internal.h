// internal.h -- launchers behind the C ABI (not exported).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace rswa {

struct DecodeArgs {
  int B, H, n;
  int64_t cap;
  int splits;
  const uint16_t* q;
  const uint16_t* pk;
  const uint16_t* pv;
  const int32_t* prefix_len;
  const uint16_t* ring_k;
  const uint16_t* ring_v;
  const int32_t* wp;
  const int32_t* fill;
  float qscale;  // softmax scale * log2(e)
  int tiles_per_item;  // P: tiles of one (sequence, head, split) item (padded with empty tiles)
  int items;           // B * H * splits
  float* out;
  float* lse;
  float* partials;   // [B*H][splits][D + 2]
  int32_t* counters; // [B*H]
  int32_t* status;
  // SR-SWA only
  const int32_t* blk_idx;
  const float* blk_logp;
  int topk;
  // FP8 prefix (E4M3 codes + per (b, h, 32-token block) scales); pk / pv unused then
  const uint8_t* pk8;
  const uint8_t* pv8;
  const float* kscale;  // [B*H][nb_cap]
  const float* vscale;
  int64_t nb_cap;
  int fp8;
  // SR-SWA chunked prefill: T queries per (sequence, head) and the chunk's output K/V
  // [B][H][T][D], read as each query's causal band; T = 1 and k_out = null for decode
  int T;
  const uint16_t* k_out;
  const uint16_t* v_out;
  // fused ring append (decode only): this step's K/V [B][H][D] join the key set as one extra
  // row, the warp that issues that row writes it into ring slot wp[b], and the launch's last
  // CTA advances wp / fill (grid_counter: a zeroed int32 in the workspace); null otherwise
  const uint16_t* k_new;
  const uint16_t* v_new;
  uint16_t* ring_k_w;
  uint16_t* ring_v_w;
  int32_t* wp_w;
  int32_t* fill_w;
  int32_t* slot_out;
  int32_t* grid_counter;
  // page2d rotary encoding inside the fused append (null rope_tok: none): this step's query
  // and key rows of sequence b are encoded at positions (rope_tok[b], rope_page[b]) on the
  // way into the attention (the query) and into the ring slot and the key set (the key)
  const int32_t* rope_tok;
  const int32_t* rope_page;
  double rope_log2_base;
  int rope_page_mod;
  // FP8 ring (decode only): E4M3 code rows [B][H][n][D] with one f32 scale per row [B][H][n]
  // for K and for V, in place of ring_k / ring_v (which are then null)
  const uint8_t* ring_k8;
  const uint8_t* ring_v8;
  const float* ring_ks;
  const float* ring_vs;
  // every pipeline wait gives up after wait_limit_ns; drop_tile >= 0 (a test of that path
  // only) makes CTA 0 skip the copy of its CTA-local tile drop_tile while still waiting on it
  uint64_t wait_limit_ns;
  int drop_tile;
  // SR-SWA with the router fused into the launch: every warp of the grid scores 64-block
  // slices of kbar against q_idx and publishes each slice sorted; the last n_fin CTAs each
  // finalise the route of their sequences (entmax threshold, top-k, ln p) into blk_idx_w /
  // blk_logp_w (tau_w nullable) and raise route_ready[b]; attention warps wait for that flag
  // before they issue a routed block's copy (token and ring tiles need no route)
  const float* q_idx;    // [B][32]
  const float* kbar;     // [B][nb_cap][32]
  float idx_scale;
  int nsl_cap;           // slices per sequence: ceil(nb_cap / 64)
  int n_fin;
  float* slice_max;      // [B][nsl_cap]
  float* slice_z;        // [B][nsl_cap][64], each slice sorted (larger score first, ties to the smaller block)
  int32_t* slice_i;      // [B][nsl_cap][64]
  int32_t* seq_count;    // [B]: slices published in this launch
  int32_t* route_ready;  // [B]: the route was published in this launch
  int32_t* blk_idx_w;    // [B][topk]
  float* blk_logp_w;
  float* tau_w;
};

// Workspace layout shared by every op: [status: 256 B][counters][partials].
struct WorkspacePlan {
  int splits, tiles_per_item, grid;
  int64_t items;
  size_t counters_off, partials_off, bytes;
};

// max_bytes > 0 restricts the split count to plans whose workspace fits that many bytes.
WorkspacePlan plan_decode_workspace(int B, int H, int64_t max_tiles, int sm_count, size_t max_bytes = 0);
int64_t decode_max_tiles_dense(int64_t cap, int n);
int decode_ctas_per_sm();  // resident decode CTAs per SM (shared-memory bound)
int64_t decode_max_tiles_sparse(int topk, int n);
int device_sm_count();

cudaError_t launch_append(int B, int H, int n, uint16_t* ring_k, uint16_t* ring_v, const uint16_t* k_new,
                          const uint16_t* v_new, int32_t* wp, int32_t* fill, int32_t* slot_out, int32_t* status,
                          cudaStream_t stream);
cudaError_t launch_decode(const DecodeArgs& a, int grid, bool sparse, cudaStream_t stream);
// Resident CTAs per SM of the decode kernel with the router fused (occupancy query), and the
// bytes of its route area in the workspace.
int routed_decode_ctas_per_sm();
size_t route_area_bytes(int B, int64_t cap);
// Ring append into an FP8 ring: each written K / V row quantised with its own scale.
cudaError_t launch_append_fp8(int B, int H, int n, uint8_t* ring_k8, uint8_t* ring_v8, float* ring_ks, float* ring_vs,
                              const uint16_t* k_new, const uint16_t* v_new, int32_t* wp, int32_t* fill,
                              int32_t* slot_out, int32_t* status, cudaStream_t stream);
// page2d rotary encoding of rows x [H][D] of q (and k when not NULL); outputs may alias inputs.
cudaError_t launch_rope(int64_t rows, int H, int D, const uint16_t* q, uint16_t* q_out, const uint16_t* k,
                        uint16_t* k_out, const int32_t* tok_pos, const int32_t* page, double base, int page_mod,
                        cudaStream_t stream);
// launch_append with the new key rotated (page2d) before it is written and the query rotated into q_out.
cudaError_t launch_append_rope(int B, int H, int n, uint16_t* ring_k, uint16_t* ring_v, const uint16_t* k_new,
                               const uint16_t* v_new, const uint16_t* q, uint16_t* q_out, const int32_t* tok_pos,
                               const int32_t* page, double base, int page_mod, int32_t* wp, int32_t* fill,
                               int32_t* slot_out, int32_t* status, cudaStream_t stream);
cudaError_t launch_quantize_prefix(int B, int H, int64_t cap, const uint16_t* pk, const uint16_t* pv,
                                   const int32_t* prefix_len, uint8_t* pk8, uint8_t* pv8, float* k_scale,
                                   float* v_scale, int32_t* status, cudaStream_t stream);
cudaError_t launch_index_pool(int B, int64_t cap, const uint16_t* k_idx, const int32_t* prefix_len, float* kbar,
                              cudaStream_t stream);
// CTAs per sequence of the router (its thread-block cluster size).
int route_cluster_size(int64_t cap);
// tokens: router queries per sequence (q_idx [B][tokens][32], outputs [B][tokens][topk])
cudaError_t launch_route(int B, int tokens, int64_t cap, const float* q_idx, const float* kbar,
                         const int32_t* prefix_len, float idx_scale, int topk, int32_t* blk_idx, float* blk_logp,
                         float* probs, float* tau, int32_t* status, cudaStream_t stream);

struct PrefillLaunch {
  int B, H, n, T;
  int64_t cap;
  const void* q;
  const void* k_out;
  const void* v_out;
  const void* pk;
  const void* pv;
  const int32_t* prefix_len;
  const void* ring_k;  // NULL: no previous chunk
  const void* ring_v;
  const int32_t* wp;
  const int32_t* fill;
  float scale;
  float* out;
  float* lse;
  int write_ring;
  void* ring_k_w;      // same buffers as ring_k/ring_v/wp/fill, written when write_ring
  void* ring_v_w;
  int32_t* wp_w;
  int32_t* fill_w;
  int32_t* status;
  int ignore_prefix;  // 1: attend to the band and the ring only (m = 0 for every sequence)
};

size_t prefill_smem_bytes();
cudaError_t launch_prefill(const PrefillLaunch& L, cudaStream_t stream);

// SR-SWA chunked prefill on tensor cores: workspace bytes beyond the status area, the grouping
// of a chunk's queries by routed block set, and the routed part merged into the band part.
size_t srswa_prefill_scratch_bytes(int B, int H, int T);
int srswa_prefill_group_rec_ints();
cudaError_t launch_srswa_group(int B, int T, int topk, int64_t cap, const int32_t* prefix_len, const int32_t* blk,
                               const float* logp, int32_t* rec, int32_t* gq, int32_t* gblk, float* gbias,
                               int32_t* counts, uint64_t* keys, int32_t* status, cudaStream_t stream);
cudaError_t launch_srswa_routed(int B, int H, int T, int topk, int64_t cap, const int32_t* prefix_len, const void* q,
                                const void* pk, const void* pv, const int32_t* rec, const int32_t* gq,
                                const float* gbias, const int32_t* counts, float scale, float* out, float* lse,
                                int32_t* status, cudaStream_t stream);

}  // namespace rswa
