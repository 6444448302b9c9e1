// Internal declarations shared by the host API and the kernels of libpv.
// Nothing here is part of the C ABI (include/pv.h is).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <atomic>

#include "../../include/pv.h"

namespace pv {

using bf16 = __nv_bfloat16;

constexpr int kMaxSteps = 8;              // denoising steps per chunk a handle may hold
constexpr int kQRows = 128;               // query rows per tensor-core tile (MMA M)
constexpr int kQTilesPerCta = 2;          // two query tiles share each K/V tile
constexpr int kOutRows = 32;               // output rows of one TMA store (one softmax warp)
constexpr int kQBlock = kQRows * kQTilesPerCta;
constexpr int kKeyTile = 128;             // keys per K/V tile (MMA N of Q K^T)
constexpr int kMaxGrid = 160;             // CTAs of one attention launch at most (>= SMs)

// ---------------------------------------------------------------- RoPE + append
struct RopeStreamDesc {
    int in_tok0;                     // first token of this stream in the packed input
    int n_tok;                       // tokens of the chunk
    int frame0;                      // latent frame of token 0
    int n_dst;                       // K/V destinations (0: none, 1: a step, steps: sink pass)
    long long qrot_row0;             // q_rot row (of D elements) of head 0, token 0
    long long dst_row0[kMaxSteps];   // K/V-region row of head 0, token 0, per destination
};

struct RopeParams {
    const bf16* q;
    const bf16* k;
    const bf16* v;
    bf16* q_rot;
    bf16* k_dst;            // K region base (store) or k_rot (dense)
    bf16* v_dst;            // V region base (store) or v head-major (dense)
    const float2* table;    // cos, sin per (axis, position, pair)
    int heads, head_dim, frame_w, frame_h;
    int pairs_t, pairs_h, pairs_w;
    int tab_h0, tab_w0;     // table offsets of the height and width blocks
    long long dst_head_stride;  // destination rows between heads
    // projection input instead of q, k, v (pv_qkv_rope_append): y f32
    // [tokens][3 * dim], ss the q / k sums of squares per token, gains g_q, g_k
    const float* y;
    const float* ss;
    const float* g_q;
    const float* g_k;
    float eps;
    int n_streams;
    RopeStreamDesc st[PV_MAX_STREAMS];
};

cudaError_t launch_rope(const RopeParams& p, int max_tok, cudaStream_t s);

// ----------------------------------------------------------------- attention
struct AttnStreamDesc {
    int n_q;             // queries of this stream (per head)
    int n_k;             // keys (per head)
    int q_row0;          // q_rot row of head 0, query 0 (per head + n_q)
    int kv_row0;         // K/V row of head 0, key 0
    int kv_head_stride;  // K/V rows between heads
    int out_tok0;        // first token row of out / lse
    int n_qb;            // query blocks of kQBlock rows
    int n_kt;            // key tiles
    int item0;           // global index of this stream's first (head, query block) item
    long long cost0;     // key tiles of all items before this stream's first
};

// One launch is a list of items (head, query block) of all streams, each
// costing n_kt key tiles, laid end to end.  Under stream-K, CTA c of `grid`
// processes one contiguous range of that list; otherwise the CTAs take whole
// items one at a time (pv_plan.cu chooses).  The whole struct plus four
// tensor maps stays under 4 KB of kernel parameters.
struct AttnParams {
    bf16* out;
    float* lse;
    float* partial;      // split-KV partial results, 4 slots per CTA (unnormalised O, m, l)
    int* counters;       // arrivals per (item, query tile); the last arriver resets to 0
    int* err;            // device error word (bounded waits that gave up)
    int heads;
    int head_dim;
    float scale_log2;    // log2(e) / sqrt(D)
    int n_streams;
    int grid;            // CTAs of the launch
    int item_aligned;    // 0: stream-K; 1: whole items handed out at run time, in
                         // list order, from counters[0] (no partial results)
    int n_items;         // items of all streams
    long long total;     // key tiles of all items
    AttnStreamDesc st[PV_MAX_STREAMS];
};

// Bytes of one partial-result slot for head dimension D.
__host__ __device__ inline size_t partial_slot_floats(int D) { return (size_t)kQRows * D + 2 * kQRows; }

cudaError_t launch_attn(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                        const CUtensorMap& to, const AttnParams& p, cudaStream_t s);

// One bounded device wait that runs out (failure-path self-test).
cudaError_t launch_wait_timeout_probe(int* err, cudaStream_t s);

// ----------------------------------------------------------------- Euler
// q, k, v projection (pv_gemm.cu): y = x w^T + b in f32 and the q / k sums of
// squares per token; tiles of 256 tokens x qkv_gemm_tile_n(dim) features.
int qkv_gemm_tile_n(int dim);
cudaError_t launch_qkv_gemm(const CUtensorMap& tx, const CUtensorMap& tw, const CUtensorMap& ty,
                            const float* bias, float* ss, int tokens, int dim, int* err,
                            cudaStream_t s);
// Destinations of the fused epilogue's TMA stores, each [rows][head_dim]
// bf16 with boxes of 32 rows x 64 features (128-byte swizzle): q_rot, the K
// region and the V region.
struct QkvOutMaps {
    CUtensorMap q, k, v;
};
// The same GEMM with the QK-Norm, RoPE and append in its epilogue (one
// cooperative launch).  ss [tokens][2][dim / tile width] takes one partial
// sum of squares per feature tile (no need to clear it); CTA c sets
// flags[c] = epoch once its partial sums are written, and the CTAs of a
// token block read them once all of its tiles' flags hold epoch (flags of
// earlier calls hold smaller values: the epoch is a 64-bit call count).  cudaErrorCooperativeLaunchTooLarge when
// its tiles cannot all be resident, there are more than kQkvFlags of them,
// or the RoPE table does not fit in shared memory beside them.
constexpr int kQkvFlags = 1024;
cudaError_t launch_qkv_fused(const CUtensorMap& tx, const CUtensorMap& tw, const float* bias,
                             float* ss, unsigned long long* flags, unsigned long long epoch,
                             int tokens, int dim, int* err, const RopeParams& rp,
                             const QkvOutMaps& om, cudaStream_t s);
bool encode_2d_map(CUtensorMap* map, const void* base, CUtensorMapDataType type, int elem_bytes,
                   long long cols, long long rows, int box_cols, int box_rows, char* err,
                   size_t errlen);
cudaError_t launch_euler(float* x, const float* v, size_t n, float dsigma, cudaStream_t s);
cudaError_t launch_euler_cfg(float* x, const float* vc, const float* vu, size_t n, float w,
                             float dsigma, cudaStream_t s);
cudaError_t launch_x0(float* x0, const float* x, const float* v, size_t n, float sigma,
                      cudaStream_t s);

// ----------------------------------------------------------------- host helpers
// Encodes a 2D bf16 tensor map over `rows` rows of `D` elements with a
// 64-element x 128-row box and the 128-byte swizzle.
bool encode_out_map(CUtensorMap* map, void* out, long long tokens, int heads, int D, char* err,
                    size_t errlen);
bool encode_rows_map(CUtensorMap* map, const void* base, long long rows, int D, char* err,
                     size_t errlen);

// Raises `kernel`'s dynamic shared-memory limit to `bytes` on the current
// device.  The attribute belongs to a device, so it is set once per device:
// `done` holds one bit per device ordinal below 64 (others set it on every
// call).  Two host threads that race here both set the same value.
template <typename K>
cudaError_t smem_limit_once(K kernel, int bytes, std::atomic<unsigned long long>& done) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const unsigned long long bit = (dev >= 0 && dev < 64) ? 1ull << dev : 0ull;
    if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return e;
    if (bit) done.fetch_or(bit, std::memory_order_release);
    return cudaSuccess;
}

// Device address, on the current device, of the fixed scratch array of
// pv_attn_dense_noalloc (its first 256 bytes hold the device error word).
cudaError_t noalloc_scratch_address(void** out);

// Records a failure for pv_last_error() and returns code.
pv_status report_error(pv_status code, const char* msg);

// Work plan for one attention launch: fills n_qb, n_kt, item0, cost0 of
// every stream and grid, total, n_items, item_aligned of p (and may reorder
// p.st).  Returns the number of CTAs, or -1 when the counters (one per item,
// at least two) do not fit.  Long items run stream-K; short items, or a
// workspace without room for the partial slots (4 per CTA), get whole items
// handed out at run time instead.
int plan_attention(AttnParams& p, int n_sm, int part_capacity, int cnt_capacity);

}  // namespace pv
