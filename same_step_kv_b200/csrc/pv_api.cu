// Host side of libpv: argument checks, the chunk schedule of each stream,
// buffer layout, tensor maps and launches.  Every entry point is extern "C"
// and returns a pv_status (include/pv.h); no C++ exception crosses the ABI.
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <map>
#include <mutex>
#include <new>
#include <vector>

#include "pv_internal.h"

using namespace pv;

namespace {

thread_local char g_err[512] = "";
thread_local pv_status g_err_code = PV_OK;

pv_status fail(pv_status code, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof(g_err), fmt, ap);
    va_end(ap);
    g_err_code = code;
    return code;
}

pv_status cuda_fail(cudaError_t e, const char* what) {
    return fail(PV_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// Surfaces a sticky or pending asynchronous error from earlier launches.
pv_status check_async(const char* what) {
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, what);
    return PV_OK;
}

bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct StreamState {
    int phase = PV_PHASE_NEW;
    int chunk = -1;
    int fill = 0;
    int slot = -1;
    int slot_frame[PV_MAX_RING];
    StreamState() { std::fill(slot_frame, slot_frame + PV_MAX_RING, -1); }
};

// Workspace layout: [error word | counters | projection flags | RoPE table |
// partial slots].
struct WsLayout {
    size_t err_off, cnt_off, flag_off, tab_off, part_off, total;
    int n_counters, n_partials, n_table;
};

constexpr int kMaxLen = 1 << 30;          // queries or keys of one sequence at most
constexpr int kMaxFrameTokens = 1 << 24;  // tokens of one latent frame at most
constexpr int kMaxFramesCfg = 1 << 20;    // RoPE table rows of the time axis at most

int tokens_per_frame(const pv_kv_config& c) { return c.frame_w * c.frame_h; }

WsLayout ws_layout(const pv_kv_config& c) {
    WsLayout w{};
    const int T = tokens_per_frame(c);
    const int max_q = c.first_frames * T;
    const int n_qb = (max_q + kQBlock - 1) / kQBlock;
    w.n_counters = c.max_streams * c.heads * n_qb * kQTilesPerCta;
    // Stream-K partial results: 4 slots per CTA, at most kMaxGrid CTAs.
    w.n_partials = 4 * kMaxGrid;
    w.n_table = c.max_frames * c.rope_pairs_t + c.frame_h * c.rope_pairs_h +
                c.frame_w * c.rope_pairs_w;
    w.err_off = 0;
    w.cnt_off = 256;
    w.flag_off = round_up(w.cnt_off + sizeof(int) * (size_t)w.n_counters, 256);
    w.tab_off = round_up(w.flag_off + sizeof(unsigned long long) * (size_t)kQkvFlags, 256);
    w.part_off = round_up(w.tab_off + sizeof(float2) * (size_t)w.n_table, 256);
    w.total = round_up(w.part_off + sizeof(float) * partial_slot_floats(c.head_dim) *
                                        (size_t)w.n_partials, 256);
    return w;
}

pv_status check_config(const pv_kv_config* c) {
    if (!c) return fail(PV_ERR_INVALID_ARG, "config is NULL");
    if (c->head_dim != 64 && c->head_dim != 128)
        return fail(PV_ERR_SHAPE, "head_dim %d: only 64 and 128 are supported", c->head_dim);
    if (c->layers < 1 || c->heads < 1 || c->frame_w < 1 || c->frame_h < 1 ||
        c->first_frames < 1 || c->max_streams < 1 || c->max_frames < 1)
        return fail(PV_ERR_SHAPE, "layers, heads, frame size, first_frames, max_streams and "
                                  "max_frames must be positive");
    if (c->ring_slots < 1 || c->ring_slots > PV_MAX_RING)
        return fail(PV_ERR_SHAPE, "ring_slots %d outside 1..%d", c->ring_slots, PV_MAX_RING);
    if (c->steps < 1 || c->steps > kMaxSteps)
        return fail(PV_ERR_SHAPE, "steps %d outside 1..%d", c->steps, kMaxSteps);
    if (c->max_streams > PV_MAX_STREAMS)
        return fail(PV_ERR_SHAPE, "max_streams %d above %d", c->max_streams, PV_MAX_STREAMS);
    if (c->rope_pairs_t < 0 || c->rope_pairs_h < 0 || c->rope_pairs_w < 0 ||
        c->rope_pairs_t + c->rope_pairs_h + c->rope_pairs_w != c->head_dim / 2)
        return fail(PV_ERR_SHAPE, "RoPE pairs %d+%d+%d must sum to head_dim/2 = %d",
                    c->rope_pairs_t, c->rope_pairs_h, c->rope_pairs_w, c->head_dim / 2);
    if (!(c->rope_theta > 1.0) || !std::isfinite(c->rope_theta))
        return fail(PV_ERR_SHAPE, "rope_theta must be finite and > 1");
    // bounds before any int product of these fields (tokens per frame, the
    // RoPE table's rows) is formed
    if ((long long)c->frame_w * c->frame_h > kMaxFrameTokens)
        return fail(PV_ERR_SHAPE, "frame of %d x %d tokens above %d", c->frame_w, c->frame_h,
                    kMaxFrameTokens);
    if (c->max_frames > kMaxFramesCfg)
        return fail(PV_ERR_SHAPE, "max_frames %d above %d", c->max_frames, kMaxFramesCfg);
    const int T = tokens_per_frame(*c);
    const long long ltot = (long long)(c->first_frames + c->ring_slots) * T;
    const long long rows = (long long)c->layers * c->steps * c->max_streams * c->heads * ltot;
    if (rows >= (1LL << 31) || (long long)c->first_frames * T * c->heads >= (1LL << 30))
        return fail(PV_ERR_SHAPE, "store of %lld rows exceeds the 2^31 rows a tensor map addresses",
                    rows);
    if (c->first_frames - 1 + 1 > c->max_frames)
        return fail(PV_ERR_SHAPE, "max_frames %d smaller than first_frames", c->max_frames);
    return PV_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000,
                                             cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = (PFN_cuTensorMapEncodeTiled_v12000)p;
    });
    return fn;
}

pv_status check_device(int* n_sm) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    int major = 0, minor = 0;
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (major != 10 || minor != 0)
        return fail(PV_ERR_UNSUPPORTED_ARCH, "device %d is sm_%d%d; libpv is built for sm_100a",
                    dev, major, minor);
    if (n_sm) cudaDeviceGetAttribute(n_sm, cudaDevAttrMultiProcessorCount, dev);
    return PV_OK;
}

}  // namespace

namespace pv {

pv_status report_error(pv_status code, const char* msg) { return fail(code, "%s", msg); }

bool encode_rows_map(CUtensorMap* map, const void* base, long long rows, int D, char* err,
                     size_t errlen) {
    auto enc = get_encode();
    if (!enc) {
        snprintf(err, errlen, "cuTensorMapEncodeTiled is not available from the driver");
        return false;
    }
    cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)D * sizeof(bf16)};
    cuuint32_t box[2] = {64, (cuuint32_t)kQRows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                     strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        snprintf(err, errlen, "cuTensorMapEncodeTiled failed (%d) for %lld rows x %d", (int)r,
                 rows, D);
        return false;
    }
    return true;
}

// The attention output out[token][head][D] (bf16) as a 3D tensor (D, heads,
// tokens) for TMA stores: a box is 64 columns of one head for 32 consecutive
// tokens (one softmax warp's rows), 128-byte swizzled like the staging buffer.
bool encode_out_map(CUtensorMap* map, void* out, long long tokens, int heads, int D, char* err,
                    size_t errlen) {
    auto enc = get_encode();
    if (!enc) {
        snprintf(err, errlen, "cuTensorMapEncodeTiled is not available from the driver");
        return false;
    }
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)heads, (cuuint64_t)tokens};
    cuuint64_t strides[2] = {(cuuint64_t)D * sizeof(bf16), (cuuint64_t)heads * D * sizeof(bf16)};
    cuuint32_t box[3] = {64, 1, (cuuint32_t)kOutRows};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, out, dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        snprintf(err, errlen, "cuTensorMapEncodeTiled failed (%d) for the output, %lld tokens x %d x %d",
                 (int)r, tokens, heads, D);
        return false;
    }
    return true;
}

bool encode_2d_map(CUtensorMap* map, const void* base, CUtensorMapDataType type, int elem_bytes,
                   long long cols, long long rows, int box_cols, int box_rows, char* err,
                   size_t errlen) {
    auto enc = get_encode();
    if (!enc) {
        snprintf(err, errlen, "cuTensorMapEncodeTiled is not available from the driver");
        return false;
    }
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)cols * elem_bytes};
    cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(map, type, 2, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        snprintf(err, errlen, "cuTensorMapEncodeTiled failed (%d) for %lld x %lld, box %d x %d",
                 (int)r, rows, cols, box_rows, box_cols);
        return false;
    }
    return true;
}

}  // namespace pv

struct pv_kv_s {
    pv_kv_config cfg{};
    int T = 0;
    int ltot = 0;
    int n_sm = 148;
    bool device = false;
    bf16* kbase = nullptr;
    bf16* vbase = nullptr;
    char* ws = nullptr;
    WsLayout wl{};
    CUtensorMap tm_k{}, tm_v{};
    // the K and V regions with 32-row boxes (stores of the fused projection)
    CUtensorMap tm_k32{}, tm_v32{};
    bool maps32 = false;
    // the last call number of the fused projection (its flags' value; 64
    // bits, so that it never comes back to a value a stale flag may hold)
    unsigned long long qkv_epoch = 0;
    std::vector<StreamState> streams;
    std::mutex mu;
    // cached tensor map of the last q_rot buffer
    const void* qmap_ptr = nullptr;
    long long qmap_rows = -1;
    // cached tensor map of the last output buffer
    CUtensorMap tm_o{};
    const void* omap_ptr = nullptr;
    long long omap_rows = -1;
    CUtensorMap tm_q{};
};

namespace {

long long region_rows(const pv_kv_s* kv) {
    const pv_kv_config& c = kv->cfg;
    return (long long)c.layers * c.steps * c.max_streams * c.heads * kv->ltot;
}

// Row (of D elements) of key 0, head 0 of (layer, step, stream) in a region.
long long base_row(const pv_kv_s* kv, int layer, int step, int stream) {
    const pv_kv_config& c = kv->cfg;
    return (((long long)layer * c.steps + step) * c.max_streams + stream) * c.heads *
           (long long)kv->ltot;
}

void derive(const pv_kv_s* kv, const StreamState& s, pv_kv_state* o) {
    const pv_kv_config& c = kv->cfg;
    o->phase = s.phase;
    o->chunk = s.chunk;
    o->fill = s.fill;
    o->slot = s.slot;
    if (s.phase == PV_PHASE_NEW) {
        o->frame0 = 0;
        o->nframes = 0;
        o->n_keys = 0;
    } else if (s.phase == PV_PHASE_FIRST || s.phase == PV_PHASE_BOOT) {
        o->frame0 = 0;
        o->nframes = c.first_frames;
        o->n_keys = c.first_frames * kv->T;
    } else {
        o->frame0 = c.first_frames - 1 + s.chunk;
        o->nframes = 1;
        o->n_keys = (c.first_frames + s.fill) * kv->T;
    }
    o->n_queries = o->nframes * kv->T;
    for (int i = 0; i < PV_MAX_RING; ++i) o->slot_frame[i] = i < c.ring_slots ? s.slot_frame[i] : -1;
}

pv_status check_streams(pv_kv kv, int n_streams, const int* streams) {
    if (n_streams < 1 || n_streams > kv->cfg.max_streams || !streams)
        return fail(PV_ERR_INVALID_ARG, "n_streams %d outside 1..%d or streams NULL", n_streams,
                    kv->cfg.max_streams);
    for (int i = 0; i < n_streams; ++i) {
        if (streams[i] < 0 || streams[i] >= kv->cfg.max_streams)
            return fail(PV_ERR_INVALID_ARG, "stream id %d outside 0..%d", streams[i],
                        kv->cfg.max_streams - 1);
        for (int j = 0; j < i; ++j)
            if (streams[j] == streams[i])
                return fail(PV_ERR_INVALID_ARG, "stream id %d listed twice", streams[i]);
    }
    return PV_OK;
}

pv_status q_map(pv_kv kv, const void* q_rot, long long rows, CUtensorMap* out) {
    if (kv->qmap_ptr != q_rot || kv->qmap_rows != rows) {
        char msg[256];
        if (!encode_rows_map(&kv->tm_q, q_rot, rows, kv->cfg.head_dim, msg, sizeof msg))
            return fail(PV_ERR_CUDA, "%s", msg);
        kv->qmap_ptr = q_rot;
        kv->qmap_rows = rows;
    }
    *out = kv->tm_q;
    return PV_OK;
}

pv_status out_map(pv_kv kv, void* out, long long tokens, CUtensorMap* map) {
    if (out != kv->omap_ptr || tokens != kv->omap_rows) {
        char msg[256];
        if (!encode_out_map(&kv->tm_o, out, tokens, kv->cfg.heads, kv->cfg.head_dim, msg, sizeof msg))
            return fail(PV_ERR_CUDA, "%s", msg);
        kv->omap_ptr = out;
        kv->omap_rows = tokens;
    }
    *map = kv->tm_o;
    return PV_OK;
}

// Shape checks and sizes shared by pv_attn_varlen_ws_bytes and pv_attn_varlen.
pv_status varlen_sizes(int n_seqs, const int* n_q, const int* n_k, int heads, int head_dim,
                       long long* tot_q, long long* tot_k, size_t* n_cnt, size_t* tiles) {
    if (!n_q || !n_k) return fail(PV_ERR_INVALID_ARG, "NULL length array");
    if (n_seqs < 1 || n_seqs > PV_MAX_STREAMS)
        return fail(PV_ERR_SHAPE, "n_seqs %d outside 1..%d", n_seqs, PV_MAX_STREAMS);
    if (heads < 1 || (head_dim != 64 && head_dim != 128))
        return fail(PV_ERR_SHAPE, "heads must be positive and head_dim 64 or 128");
    *tot_q = *tot_k = 0;
    *n_cnt = *tiles = 0;
    for (int i = 0; i < n_seqs; ++i) {
        if (n_q[i] < 0 || n_k[i] < 0 || (n_q[i] > 0 && n_k[i] == 0))
            return fail(PV_ERR_SHAPE, "sequence %d: n_q %d, n_k %d (queries need keys)", i, n_q[i],
                        n_k[i]);
        if (n_q[i] > kMaxLen || n_k[i] > kMaxLen)
            return fail(PV_ERR_SHAPE, "sequence %d: n_q %d, n_k %d above %d", i, n_q[i], n_k[i],
                        kMaxLen);
        const size_t qb = (n_q[i] + kQBlock - 1) / kQBlock;
        *n_cnt += (size_t)heads * qb * kQTilesPerCta;
        *tiles += (size_t)heads * qb * ((n_k[i] + kKeyTile - 1) / kKeyTile);
        *tot_q += n_q[i];
        *tot_k += n_k[i];
    }
    if (*tot_q * heads >= (1LL << 31) || *tot_k * heads >= (1LL << 31))
        return fail(PV_ERR_SHAPE, "too many rows for a tensor map");
    return PV_OK;
}
}  // namespace

extern "C" {

const char* pv_version(void) { return "pv 0.1.0 (sm_100a)"; }

pv_status pv_last_error(char* buf, size_t len) {
    if (buf && len) {
        strncpy(buf, g_err, len - 1);
        buf[len - 1] = 0;
    }
    return g_err_code;
}

pv_status pv_kv_required_bytes(const pv_kv_config* cfg, size_t* kv_bytes, size_t* ws_bytes) {
    pv_status st = check_config(cfg);
    if (st) return st;
    if (!kv_bytes || !ws_bytes) return fail(PV_ERR_INVALID_ARG, "output pointer is NULL");
    const int T = tokens_per_frame(*cfg);
    const size_t ltot = (size_t)(cfg->first_frames + cfg->ring_slots) * T;
    *kv_bytes = 2 * (size_t)cfg->layers * cfg->steps * cfg->max_streams * cfg->heads * ltot *
                cfg->head_dim * sizeof(bf16);
    *ws_bytes = ws_layout(*cfg).total;
    return PV_OK;
}

pv_status pv_kv_init(pv_kv* out, const pv_kv_config* cfg, void* kv_dev, size_t kv_bytes,
                     void* ws_dev, size_t ws_bytes) {
    if (!out) return fail(PV_ERR_INVALID_ARG, "out handle pointer is NULL");
    *out = nullptr;
    pv_status st = check_config(cfg);
    if (st) return st;
    const bool bookkeeping_only = (kv_dev == nullptr && ws_dev == nullptr);
    if (!bookkeeping_only && (!kv_dev || !ws_dev))
        return fail(PV_ERR_INVALID_ARG, "pass both device buffers, or neither");
    size_t need_kv = 0, need_ws = 0;
    pv_kv_required_bytes(cfg, &need_kv, &need_ws);
    pv_kv_s* kv = new (std::nothrow) pv_kv_s();
    if (!kv) return fail(PV_ERR_CAPACITY, "host allocation failed");
    kv->cfg = *cfg;
    kv->T = tokens_per_frame(*cfg);
    kv->ltot = (cfg->first_frames + cfg->ring_slots) * kv->T;
    kv->streams.resize(cfg->max_streams);
    kv->wl = ws_layout(*cfg);
    if (!bookkeeping_only) {
        if (kv_bytes < need_kv || ws_bytes < need_ws) {
            delete kv;
            return fail(PV_ERR_CAPACITY, "buffers of %zu / %zu bytes, need %zu / %zu", kv_bytes,
                        ws_bytes, need_kv, need_ws);
        }
        if (!aligned(kv_dev, 256) || !aligned(ws_dev, 256)) {
            delete kv;
            return fail(PV_ERR_INVALID_ARG, "device buffers must be 256-byte aligned");
        }
        if ((st = check_device(&kv->n_sm))) {
            delete kv;
            return st;
        }
        kv->device = true;
        kv->kbase = (bf16*)kv_dev;
        kv->vbase = kv->kbase + (size_t)region_rows(kv) * cfg->head_dim;
        kv->ws = (char*)ws_dev;
        // RoPE table, fp64 on the host, stored as f32 (cos, sin).
        const pv_kv_config& c = *cfg;
        std::vector<float2> tab(kv->wl.n_table);
        auto fill_axis = [&](int base, int npos, int npairs) {
            for (int p = 0; p < npos; ++p)
                for (int k = 0; k < npairs; ++k) {
                    const double freq = std::pow(c.rope_theta, -2.0 * k / (2.0 * npairs));
                    const double a = p * freq;
                    tab[base + p * npairs + k] = make_float2((float)std::cos(a), (float)std::sin(a));
                }
        };
        fill_axis(0, c.max_frames, c.rope_pairs_t);
        fill_axis(c.max_frames * c.rope_pairs_t, c.frame_h, c.rope_pairs_h);
        fill_axis(c.max_frames * c.rope_pairs_t + c.frame_h * c.rope_pairs_h, c.frame_w,
                  c.rope_pairs_w);
        cudaError_t e = cudaMemset(kv_dev, 0, need_kv);
        if (e == cudaSuccess) e = cudaMemset(ws_dev, 0, need_ws);
        if (e == cudaSuccess)
            e = cudaMemcpy(kv->ws + kv->wl.tab_off, tab.data(), sizeof(float2) * tab.size(),
                           cudaMemcpyHostToDevice);
        if (e != cudaSuccess) {
            delete kv;
            return cuda_fail(e, "initialising the store");
        }
        char msg[256];
        if (!encode_rows_map(&kv->tm_k, kv->kbase, region_rows(kv), c.head_dim, msg, sizeof msg) ||
            !encode_rows_map(&kv->tm_v, kv->vbase, region_rows(kv), c.head_dim, msg, sizeof msg)) {
            delete kv;
            return fail(PV_ERR_CUDA, "%s", msg);
        }
        // without them pv_qkv_rope_append takes its two-launch path
        kv->maps32 = region_rows(kv) < (1LL << 31) &&
                     encode_2d_map(&kv->tm_k32, kv->kbase, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                                   c.head_dim, region_rows(kv), 64, 32, msg, sizeof msg) &&
                     encode_2d_map(&kv->tm_v32, kv->vbase, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                                   c.head_dim, region_rows(kv), 64, 32, msg, sizeof msg);
    }
    *out = kv;
    return PV_OK;
}

pv_status pv_kv_destroy(pv_kv kv) {
    delete kv;
    return PV_OK;
}

pv_status pv_kv_begin_chunk(pv_kv kv, int stream, int nframes) {
    if (!kv) return fail(PV_ERR_INVALID_ARG, "handle is NULL");
    if (stream < 0 || stream >= kv->cfg.max_streams)
        return fail(PV_ERR_INVALID_ARG, "stream %d outside 0..%d", stream, kv->cfg.max_streams - 1);
    std::lock_guard<std::mutex> lock(kv->mu);
    StreamState& s = kv->streams[stream];
    const pv_kv_config& c = kv->cfg;
    switch (s.phase) {
        case PV_PHASE_NEW:
            if (nframes != c.first_frames)
                return fail(PV_ERR_STATE, "the first chunk holds %d frames, not %d",
                            c.first_frames, nframes);
            s.phase = PV_PHASE_FIRST;
            s.chunk = 0;
            return PV_OK;
        case PV_PHASE_FIRST:
            return fail(PV_ERR_STATE, "stream %d: run the sink pass (PV_STEP_SINK) before chunk 1",
                        stream);
        default:
            if (nframes != 1)
                return fail(PV_ERR_STATE, "chunks after the first hold 1 frame, not %d", nframes);
            if (c.first_frames + s.chunk + 1 > c.max_frames)
                return fail(PV_ERR_CAPACITY, "chunk %d would reach latent frame %d >= max_frames %d",
                            s.chunk + 1, c.first_frames + s.chunk, c.max_frames);
            s.phase = PV_PHASE_STEADY;
            s.chunk += 1;
            s.slot = (s.chunk - 1) % c.ring_slots;
            s.fill = std::min(s.chunk, c.ring_slots);
            s.slot_frame[s.slot] = c.first_frames - 1 + s.chunk;
            return PV_OK;
    }
}

pv_status pv_kv_begin_sink(pv_kv kv, int stream) {
    if (!kv) return fail(PV_ERR_INVALID_ARG, "handle is NULL");
    if (stream < 0 || stream >= kv->cfg.max_streams)
        return fail(PV_ERR_INVALID_ARG, "stream %d outside 0..%d", stream, kv->cfg.max_streams - 1);
    std::lock_guard<std::mutex> lock(kv->mu);
    StreamState& s = kv->streams[stream];
    if (s.phase != PV_PHASE_FIRST)
        return fail(PV_ERR_STATE, "stream %d: the sink pass follows the first chunk (phase %d)",
                    stream, s.phase);
    s.phase = PV_PHASE_BOOT;
    return PV_OK;
}

pv_status pv_kv_get_state(pv_kv kv, int stream, pv_kv_state* out) {
    if (!kv || !out) return fail(PV_ERR_INVALID_ARG, "handle or output is NULL");
    if (stream < 0 || stream >= kv->cfg.max_streams)
        return fail(PV_ERR_INVALID_ARG, "stream %d outside 0..%d", stream, kv->cfg.max_streams - 1);
    std::lock_guard<std::mutex> lock(kv->mu);
    derive(kv, kv->streams[stream], out);
    return PV_OK;
}

pv_status pv_kv_set_state(pv_kv kv, int stream, const pv_kv_state* st) {
    if (!kv || !st) return fail(PV_ERR_INVALID_ARG, "handle or state is NULL");
    if (stream < 0 || stream >= kv->cfg.max_streams)
        return fail(PV_ERR_INVALID_ARG, "stream %d outside 0..%d", stream, kv->cfg.max_streams - 1);
    const pv_kv_config& c = kv->cfg;
    StreamState s;
    s.phase = st->phase;
    s.chunk = st->chunk;
    switch (st->phase) {
        case PV_PHASE_NEW:
            if (st->chunk != -1) return fail(PV_ERR_STATE, "NEW state must have chunk -1");
            break;
        case PV_PHASE_FIRST:
        case PV_PHASE_BOOT:
            if (st->chunk != 0) return fail(PV_ERR_STATE, "first-chunk state must have chunk 0");
            break;
        case PV_PHASE_STEADY:
            if (st->chunk < 1 || c.first_frames - 1 + st->chunk >= c.max_frames)
                return fail(PV_ERR_STATE, "steady state chunk %d out of range", st->chunk);
            s.slot = (st->chunk - 1) % c.ring_slots;
            s.fill = std::min(st->chunk, c.ring_slots);
            // slot i holds the latest chunk j' <= chunk with (j'-1) mod R == i
            for (int i = 0; i < c.ring_slots; ++i) {
                int last = st->chunk - ((st->chunk - 1 - i) % c.ring_slots + c.ring_slots) % c.ring_slots;
                s.slot_frame[i] = last >= 1 ? c.first_frames - 1 + last : -1;
            }
            break;
        default:
            return fail(PV_ERR_STATE, "unknown phase %d", st->phase);
    }
    std::lock_guard<std::mutex> lock(kv->mu);
    kv->streams[stream] = s;
    return PV_OK;
}

pv_status pv_kv_row_offset(pv_kv kv, int layer, int step, int stream, int head, int key,
                           size_t* k_elem, size_t* v_elem) {
    if (!kv || !k_elem || !v_elem) return fail(PV_ERR_INVALID_ARG, "NULL argument");
    const pv_kv_config& c = kv->cfg;
    if (layer < 0 || layer >= c.layers || step < 0 || step >= c.steps || stream < 0 ||
        stream >= c.max_streams || head < 0 || head >= c.heads || key < 0 || key >= kv->ltot)
        return fail(PV_ERR_INVALID_ARG, "index outside the store");
    const long long row = base_row(kv, layer, step, stream) + (long long)head * kv->ltot + key;
    *k_elem = (size_t)row * c.head_dim;
    *v_elem = (size_t)(region_rows(kv) + row) * c.head_dim;
    return PV_OK;
}

}  // extern "C"

namespace {
// RoPE / append parameters of the listed streams at (layer, step): the
// checks and the destinations that pv_rope_append and pv_qkv_rope_append share.
// Sets *tokens (all streams) and *max_tok.
pv_status rope_params(pv_kv kv, int n_streams, const int* streams, int layer, int step,
                      RopeParams* pp, int* tokens, int* max_tok) {
    pv_status st = check_streams(kv, n_streams, streams);
    if (st) return st;
    const pv_kv_config& c = kv->cfg;
    if (layer < 0 || layer >= c.layers) return fail(PV_ERR_INVALID_ARG, "layer %d out of range", layer);
    if (!(step == PV_STEP_SINK || (step >= 0 && step < c.steps)))
        return fail(PV_ERR_INVALID_ARG, "step %d is neither 0..%d nor PV_STEP_SINK", step, c.steps - 1);
    // validate every stream before changing any state
    for (int i = 0; i < n_streams; ++i) {
        const StreamState& s = kv->streams[streams[i]];
        if (step == PV_STEP_SINK) {
            if (s.phase != PV_PHASE_BOOT)
                return fail(PV_ERR_STATE, "stream %d: call pv_kv_begin_sink before the sink pass",
                            streams[i]);
        } else if (s.phase != PV_PHASE_FIRST && s.phase != PV_PHASE_STEADY) {
            return fail(PV_ERR_STATE, "stream %d: no denoising step in phase %d", streams[i], s.phase);
        }
    }
    RopeParams& p = *pp;
    p.k_dst = kv->kbase;
    p.v_dst = kv->vbase;
    p.table = (const float2*)(kv->ws + kv->wl.tab_off);
    p.heads = c.heads;
    p.head_dim = c.head_dim;
    p.frame_w = c.frame_w;
    p.frame_h = c.frame_h;
    p.pairs_t = c.rope_pairs_t;
    p.pairs_h = c.rope_pairs_h;
    p.pairs_w = c.rope_pairs_w;
    p.tab_h0 = c.max_frames * c.rope_pairs_t;
    p.tab_w0 = p.tab_h0 + c.frame_h * c.rope_pairs_h;
    p.dst_head_stride = kv->ltot;
    p.n_streams = n_streams;
    int tok = 0, mt = 0;
    for (int i = 0; i < n_streams; ++i) {
        StreamState& s = kv->streams[streams[i]];
        pv_kv_state d;
        derive(kv, s, &d);
        RopeStreamDesc& sd = p.st[i];
        sd.in_tok0 = tok;
        sd.n_tok = d.n_queries;
        sd.frame0 = d.frame0;
        sd.qrot_row0 = (long long)c.heads * tok;
        if (step == PV_STEP_SINK) {
            sd.n_dst = c.steps;
            for (int s2 = 0; s2 < c.steps; ++s2) sd.dst_row0[s2] = base_row(kv, layer, s2, streams[i]);
        } else if (s.phase == PV_PHASE_FIRST) {
            sd.n_dst = 1;
            sd.dst_row0[0] = base_row(kv, layer, step, streams[i]);
        } else {
            sd.n_dst = 1;
            sd.dst_row0[0] = base_row(kv, layer, step, streams[i]) +
                             (long long)(c.first_frames + s.slot) * kv->T;
        }
        tok += d.n_queries;
        mt = std::max(mt, d.n_queries);
    }
    *tokens = tok;
    *max_tok = mt;
    return PV_OK;
}

// Workspace of pv_qkv_rope_append: y f32 [tokens][3 * dim], then the sums of
// squares f32 [tokens][2][dim / tile width] (the fused launch writes one
// partial sum per feature tile; the two-launch path adds into [tokens][2]),
// each part 256-byte aligned.
size_t qkv_y_bytes(long long tokens, int dim) { return round_up((size_t)tokens * 3 * dim * 4, 256); }
size_t qkv_ss_bytes(long long tokens, int dim) {
    const int bn = qkv_gemm_tile_n(dim);
    return round_up((size_t)tokens * 2 * (bn ? dim / bn : 1) * 4, 256);
}
}  // namespace

extern "C" {

pv_status pv_rope_append(pv_kv kv, int n_streams, const int* streams, int layer, int step,
                         const void* q, const void* k, const void* v, void* q_rot,
                         void* cuda_stream) {
    if (!kv) return fail(PV_ERR_INVALID_ARG, "handle is NULL");
    if (!kv->device) return fail(PV_ERR_STATE, "bookkeeping-only handle has no device buffers");
    if (!q || !k || !v || !q_rot) return fail(PV_ERR_INVALID_ARG, "NULL tensor pointer");
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(q_rot, 16))
        return fail(PV_ERR_INVALID_ARG, "tensors must be 16-byte aligned");
    pv_status st;
    if ((st = check_async("an earlier launch"))) return st;
    std::lock_guard<std::mutex> lock(kv->mu);
    RopeParams p{};
    int tok = 0, max_tok = 0;
    if ((st = rope_params(kv, n_streams, streams, layer, step, &p, &tok, &max_tok))) return st;
    p.q = (const bf16*)q;
    p.k = (const bf16*)k;
    p.v = (const bf16*)v;
    p.q_rot = (bf16*)q_rot;
    cudaError_t e = launch_rope(p, max_tok, (cudaStream_t)cuda_stream);
    if (e != cudaSuccess) return cuda_fail(e, "rope_append launch");
    return PV_OK;
}

pv_status pv_qkv_ws_bytes(int tokens, int dim, size_t* ws_bytes) {
    if (!ws_bytes) return fail(PV_ERR_INVALID_ARG, "output pointer is NULL");
    if (tokens < 1 || dim < 64 || dim % 64 != 0)
        return fail(PV_ERR_SHAPE, "tokens must be positive and dim a multiple of 64");
    *ws_bytes = qkv_y_bytes(tokens, dim) + qkv_ss_bytes(tokens, dim);
    return PV_OK;
}

pv_status pv_qkv_rope_append(pv_kv kv, int n_streams, const int* streams, int layer, int step,
                             const void* x, const void* w, const float* bias, const float* g_q,
                             const float* g_k, float eps, void* q_rot, void* ws, size_t ws_bytes,
                             void* cuda_stream) {
    if (!kv) return fail(PV_ERR_INVALID_ARG, "handle is NULL");
    if (!kv->device) return fail(PV_ERR_STATE, "bookkeeping-only handle has no device buffers");
    if (!x || !w || !bias || !g_q || !g_k || !q_rot || !ws)
        return fail(PV_ERR_INVALID_ARG, "NULL pointer");
    if (!aligned(x, 16) || !aligned(w, 16) || !aligned(q_rot, 16) || !aligned(ws, 256) ||
        !aligned(bias, 16) || !aligned(g_q, 16) || !aligned(g_k, 16))
        return fail(PV_ERR_INVALID_ARG, "x, w, q_rot, bias, g_q, g_k 16-byte, ws 256-byte aligned");
    if (!(eps > 0.f) || !std::isfinite(eps)) return fail(PV_ERR_INVALID_ARG, "eps must be > 0");
    const pv_kv_config& c = kv->cfg;
    const int dim = c.heads * c.head_dim;
    if (qkv_gemm_tile_n(dim) == 0)
        return fail(PV_ERR_SHAPE, "heads * head_dim = %d is not a multiple of 64", dim);
    pv_status st;
    if ((st = check_async("an earlier launch"))) return st;
    std::lock_guard<std::mutex> lock(kv->mu);
    RopeParams p{};
    int tok = 0, max_tok = 0;
    if ((st = rope_params(kv, n_streams, streams, layer, step, &p, &tok, &max_tok))) return st;
    size_t need = 0;
    pv_qkv_ws_bytes(tok, dim, &need);
    if (ws_bytes < need)
        return fail(PV_ERR_CAPACITY, "workspace of %zu bytes, need %zu", ws_bytes, need);
    float* y = (float*)ws;
    float* ss = (float*)((char*)ws + qkv_y_bytes(tok, dim));
    CUtensorMap tx, tw, ty;
    char msg[256];
    const int bn = qkv_gemm_tile_n(dim);
    if (!encode_2d_map(&tx, x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, dim, tok, 64, 128, msg,
                       sizeof msg) ||
        !encode_2d_map(&tw, w, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, dim, 3LL * dim, 64, bn, msg,
                       sizeof msg) ||
        !encode_2d_map(&ty, y, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, 3LL * dim, tok, 32, 32, msg,
                       sizeof msg))
        return fail(PV_ERR_CUDA, "%s", msg);
    cudaStream_t s = (cudaStream_t)cuda_stream;
    int* err = (int*)(kv->ws + kv->wl.err_off);
    cudaError_t e;
    p.y = y;
    p.ss = ss;
    p.g_q = g_q;
    p.g_k = g_k;
    p.eps = eps;
    p.q_rot = (bf16*)q_rot;
    // one launch when every tile of the GEMM can be resident at once (the
    // steady chunk's 880 tokens: 144 CTAs) and the rows fit TMA's 32-bit
    // coordinates; else the GEMM writes y and the RoPE / append kernel
    // reads it back
    const long long qrows = (long long)c.heads * tok;
    QkvOutMaps om;
    if (kv->maps32 && qrows < (1LL << 31) &&
        encode_2d_map(&om.q, q_rot, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, c.head_dim, qrows, 64, 32,
                      msg, sizeof msg)) {
        om.k = kv->tm_k32;
        om.v = kv->tm_v32;
        // a new value for the flags of this call (0 is the cleared state)
        const unsigned long long epoch = kv->qkv_epoch + 1;
        unsigned long long* flags = (unsigned long long*)(kv->ws + kv->wl.flag_off);
        e = launch_qkv_fused(tx, tw, bias, ss, flags, epoch, tok, dim, err, p, om, s);
        if (e == cudaSuccess) {
            kv->qkv_epoch = epoch;
            return PV_OK;
        }
        if (e != cudaErrorCooperativeLaunchTooLarge) return cuda_fail(e, "qkv fused launch");
    }
    e = cudaMemsetAsync(ss, 0, (size_t)tok * 2 * sizeof(float), s);
    if (e != cudaSuccess) return cuda_fail(e, "clearing the sums of squares");
    e = launch_qkv_gemm(tx, tw, ty, bias, ss, tok, dim, err, s);
    if (e != cudaSuccess) return cuda_fail(e, "qkv projection launch");
    e = launch_rope(p, max_tok, s);
    if (e != cudaSuccess) return cuda_fail(e, "qkv rope_append launch");
    return PV_OK;
}

pv_status pv_chunk_attn(pv_kv kv, int n_streams, const int* streams, int layer, int step,
                        const void* q_rot, void* out, float* lse, void* cuda_stream) {
    if (!kv) return fail(PV_ERR_INVALID_ARG, "handle is NULL");
    if (!kv->device) return fail(PV_ERR_STATE, "bookkeeping-only handle has no device buffers");
    pv_status st = check_streams(kv, n_streams, streams);
    if (st) return st;
    const pv_kv_config& c = kv->cfg;
    if (layer < 0 || layer >= c.layers) return fail(PV_ERR_INVALID_ARG, "layer %d out of range", layer);
    if (!(step == PV_STEP_SINK || (step >= 0 && step < c.steps)))
        return fail(PV_ERR_INVALID_ARG, "step %d is neither 0..%d nor PV_STEP_SINK", step, c.steps - 1);
    if (!q_rot || !out) return fail(PV_ERR_INVALID_ARG, "NULL tensor pointer");
    if (!aligned(q_rot, 16) || !aligned(out, 16) || (lse && !aligned(lse, 4)))
        return fail(PV_ERR_INVALID_ARG, "tensors must be 16-byte aligned");
    if ((st = check_async("an earlier launch"))) return st;

    std::lock_guard<std::mutex> lock(kv->mu);
    AttnParams p{};
    p.out = (bf16*)out;
    p.lse = lse;
    p.partial = (float*)(kv->ws + kv->wl.part_off);
    p.counters = (int*)(kv->ws + kv->wl.cnt_off);
    p.err = (int*)(kv->ws + kv->wl.err_off);
    p.heads = c.heads;
    p.head_dim = c.head_dim;
    p.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)c.head_dim));
    p.n_streams = n_streams;
    int tok = 0;
    for (int i = 0; i < n_streams; ++i) {
        const StreamState& s = kv->streams[streams[i]];
        if (step == PV_STEP_SINK) {
            if (s.phase != PV_PHASE_BOOT)
                return fail(PV_ERR_STATE, "stream %d: sink attention needs the sink pass first",
                            streams[i]);
        } else if (s.phase != PV_PHASE_FIRST && s.phase != PV_PHASE_STEADY) {
            return fail(PV_ERR_STATE, "stream %d: no denoising step in phase %d", streams[i], s.phase);
        }
        pv_kv_state d;
        derive(kv, s, &d);
        AttnStreamDesc& a = p.st[i];
        a.n_q = d.n_queries;
        a.n_k = d.n_keys;
        a.q_row0 = c.heads * tok;
        a.kv_row0 = (int)base_row(kv, layer, step == PV_STEP_SINK ? 0 : step, streams[i]);
        a.kv_head_stride = kv->ltot;
        a.out_tok0 = tok;
        tok += d.n_queries;
    }
    if (plan_attention(p, kv->n_sm, kv->wl.n_partials, kv->wl.n_counters) < 0)
        return fail(PV_ERR_CAPACITY, "attention plan exceeds the workspace");
    CUtensorMap tq, to;
    if ((st = q_map(kv, q_rot, (long long)c.heads * tok, &tq))) return st;
    if ((st = out_map(kv, out, tok, &to))) return st;
    cudaError_t e = launch_attn(tq, kv->tm_k, kv->tm_v, to, p, (cudaStream_t)cuda_stream);
    if (e != cudaSuccess) return cuda_fail(e, "chunk_attn launch");
    return PV_OK;
}

pv_status pv_rope_dense(pv_kv kv, int n_tokens, int frame0, const void* q, const void* k,
                        const void* v, void* q_rot, void* k_rot, void* v_hm, void* cuda_stream) {
    if (!kv) return fail(PV_ERR_INVALID_ARG, "handle is NULL");
    if (!kv->device) return fail(PV_ERR_STATE, "bookkeeping-only handle has no device buffers");
    const pv_kv_config& c = kv->cfg;
    if (n_tokens < 1 || n_tokens % kv->T != 0)
        return fail(PV_ERR_SHAPE, "n_tokens %d is not a positive multiple of %d", n_tokens, kv->T);
    if (frame0 < 0 || (long long)frame0 + n_tokens / kv->T > c.max_frames)
        return fail(PV_ERR_SHAPE, "frames %d..%d outside the RoPE table (max_frames %d)", frame0,
                    frame0 + n_tokens / kv->T - 1, c.max_frames);
    if ((long long)n_tokens * c.heads >= (1LL << 31))
        return fail(PV_ERR_SHAPE, "too many tokens");
    if (!q || !k || !v || !q_rot || !k_rot || !v_hm) return fail(PV_ERR_INVALID_ARG, "NULL tensor");
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(q_rot, 16) ||
        !aligned(k_rot, 16) || !aligned(v_hm, 16))
        return fail(PV_ERR_INVALID_ARG, "tensors must be 16-byte aligned");
    pv_status st;
    if ((st = check_async("an earlier launch"))) return st;
    RopeParams p{};
    p.q = (const bf16*)q;
    p.k = (const bf16*)k;
    p.v = (const bf16*)v;
    p.q_rot = (bf16*)q_rot;
    p.k_dst = (bf16*)k_rot;
    p.v_dst = (bf16*)v_hm;
    p.table = (const float2*)(kv->ws + kv->wl.tab_off);
    p.heads = c.heads;
    p.head_dim = c.head_dim;
    p.frame_w = c.frame_w;
    p.frame_h = c.frame_h;
    p.pairs_t = c.rope_pairs_t;
    p.pairs_h = c.rope_pairs_h;
    p.pairs_w = c.rope_pairs_w;
    p.tab_h0 = c.max_frames * c.rope_pairs_t;
    p.tab_w0 = p.tab_h0 + c.frame_h * c.rope_pairs_h;
    p.dst_head_stride = n_tokens;
    p.n_streams = 1;
    p.st[0].in_tok0 = 0;
    p.st[0].n_tok = n_tokens;
    p.st[0].frame0 = frame0;
    p.st[0].qrot_row0 = 0;
    p.st[0].n_dst = 1;
    p.st[0].dst_row0[0] = 0;
    cudaError_t e = launch_rope(p, n_tokens, (cudaStream_t)cuda_stream);
    if (e != cudaSuccess) return cuda_fail(e, "rope_dense launch");
    return PV_OK;
}

pv_status pv_attn_dense_ws_bytes(int n_q, int n_k, int heads, int head_dim, size_t* ws_bytes) {
    if (!ws_bytes) return fail(PV_ERR_INVALID_ARG, "output pointer is NULL");
    if (n_q < 1 || n_k < 1 || heads < 1 || (head_dim != 64 && head_dim != 128))
        return fail(PV_ERR_SHAPE, "bad dense attention shape");
    if (n_q > kMaxLen || n_k > kMaxLen)
        return fail(PV_ERR_SHAPE, "n_q %d or n_k %d above %d", n_q, n_k, kMaxLen);
    const size_t n_qb = (n_q + kQBlock - 1) / kQBlock;
    const size_t n_cnt = (size_t)heads * n_qb * kQTilesPerCta;
    const size_t tiles = (size_t)heads * n_qb * ((n_k + kKeyTile - 1) / kKeyTile);
    const size_t n_part = 4 * std::min<size_t>(kMaxGrid, tiles);
    *ws_bytes = 256 + round_up(n_cnt * sizeof(int), 256) +
                n_part * partial_slot_floats(head_dim) * sizeof(float);
    return PV_OK;
}

pv_status pv_attn_dense(const void* q, const void* k, const void* v, int n_q, int n_k, int heads,
                        int head_dim, void* out, float* lse, void* ws, size_t ws_bytes,
                        void* cuda_stream) {
    if (!q || !k || !v || !out) return fail(PV_ERR_INVALID_ARG, "NULL tensor pointer");
    if (n_q < 1 || n_k < 1 || heads < 1 || (head_dim != 64 && head_dim != 128))
        return fail(PV_ERR_SHAPE, "n_q, n_k, heads must be positive and head_dim 64 or 128");
    if (n_q > kMaxLen || n_k > kMaxLen)
        return fail(PV_ERR_SHAPE, "n_q %d or n_k %d above %d", n_q, n_k, kMaxLen);
    if ((long long)n_q * heads >= (1LL << 31) || (long long)n_k * heads >= (1LL << 31))
        return fail(PV_ERR_SHAPE, "too many rows for a tensor map");
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16))
        return fail(PV_ERR_INVALID_ARG, "tensors must be 16-byte aligned");
    size_t need = 0;
    pv_attn_dense_ws_bytes(n_q, n_k, heads, head_dim, &need);
    if (!ws || ws_bytes < need || !aligned(ws, 256))
        return fail(PV_ERR_CAPACITY, "workspace of %zu bytes at %p, need %zu (256-byte aligned)",
                    ws_bytes, ws, need);
    pv_status st;
    if ((st = check_async("an earlier launch"))) return st;
    int n_sm = 148;
    if ((st = check_device(&n_sm))) return st;
    const size_t n_qb = (n_q + kQBlock - 1) / kQBlock;
    const int n_cnt = (int)((size_t)heads * n_qb * kQTilesPerCta);
    const size_t tiles = (size_t)heads * n_qb * ((n_k + kKeyTile - 1) / kKeyTile);
    const int n_part = (int)(4 * std::min<size_t>(kMaxGrid, tiles));
    AttnParams p{};
    p.out = (bf16*)out;
    p.lse = lse;
    p.err = (int*)ws;
    p.counters = (int*)((char*)ws + 256);
    p.partial = (float*)((char*)ws + 256 + round_up((size_t)n_cnt * sizeof(int), 256));
    p.heads = heads;
    p.head_dim = head_dim;
    p.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)head_dim));
    p.n_streams = 1;
    AttnStreamDesc& a = p.st[0];
    a.n_q = n_q;
    a.n_k = n_k;
    a.q_row0 = 0;
    a.kv_row0 = 0;
    a.kv_head_stride = n_k;
    a.out_tok0 = 0;
    if (plan_attention(p, n_sm, n_part, n_cnt) < 0)
        return fail(PV_ERR_CAPACITY, "attention plan exceeds the workspace");
    CUtensorMap tq, tk, tv;
    char msg[256];
    CUtensorMap to;
    if (!encode_rows_map(&tq, q, (long long)heads * n_q, head_dim, msg, sizeof msg) ||
        !encode_rows_map(&tk, k, (long long)heads * n_k, head_dim, msg, sizeof msg) ||
        !encode_rows_map(&tv, v, (long long)heads * n_k, head_dim, msg, sizeof msg) ||
        !encode_out_map(&to, out, n_q, heads, head_dim, msg, sizeof msg))
        return fail(PV_ERR_CUDA, "%s", msg);
    cudaError_t e = launch_attn(tq, tk, tv, to, p, (cudaStream_t)cuda_stream);
    if (e != cudaSuccess) return cuda_fail(e, "attn_dense launch");
    return PV_OK;
}

pv_status pv_attn_varlen_ws_bytes(int n_seqs, const int* n_q, const int* n_k, int heads,
                                  int head_dim, size_t* ws_bytes) {
    if (!ws_bytes) return fail(PV_ERR_INVALID_ARG, "output pointer is NULL");
    long long tq = 0, tk = 0;
    size_t n_cnt = 0, tiles = 0;
    pv_status st = varlen_sizes(n_seqs, n_q, n_k, heads, head_dim, &tq, &tk, &n_cnt, &tiles);
    if (st) return st;
    const size_t n_part = 4 * std::min<size_t>(kMaxGrid, std::max<size_t>(tiles, 1));
    *ws_bytes = 256 + round_up(std::max<size_t>(n_cnt, 1) * sizeof(int), 256) +
                n_part * partial_slot_floats(head_dim) * sizeof(float);
    return PV_OK;
}

pv_status pv_attn_varlen(const void* q, const void* k, const void* v, int n_seqs, const int* n_q,
                         const int* n_k, int heads, int head_dim, void* out, float* lse, void* ws,
                         size_t ws_bytes, void* cuda_stream) {
    long long tot_q = 0, tot_k = 0;
    size_t n_cnt = 0, tiles = 0;
    pv_status st = varlen_sizes(n_seqs, n_q, n_k, heads, head_dim, &tot_q, &tot_k, &n_cnt, &tiles);
    if (st) return st;
    if (tot_q == 0) return PV_OK;  // no queries: nothing to compute
    if (!q || !k || !v || !out) return fail(PV_ERR_INVALID_ARG, "NULL tensor pointer");
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16))
        return fail(PV_ERR_INVALID_ARG, "tensors must be 16-byte aligned");
    size_t need = 0;
    pv_attn_varlen_ws_bytes(n_seqs, n_q, n_k, heads, head_dim, &need);
    if (!ws || ws_bytes < need || !aligned(ws, 256))
        return fail(PV_ERR_CAPACITY, "workspace of %zu bytes at %p, need %zu (256-byte aligned)",
                    ws_bytes, ws, need);
    if ((st = check_async("an earlier launch"))) return st;
    int n_sm = 148;
    if ((st = check_device(&n_sm))) return st;
    const int n_part = (int)(4 * std::min<size_t>(kMaxGrid, tiles));
    AttnParams p{};
    p.out = (bf16*)out;
    p.lse = lse;
    p.err = (int*)ws;
    p.counters = (int*)((char*)ws + 256);
    p.partial = (float*)((char*)ws + 256 + round_up(n_cnt * sizeof(int), 256));
    p.heads = heads;
    p.head_dim = head_dim;
    p.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)head_dim));
    // sequence i: queries at head-major rows heads*qoff + h*n_q[i], keys at
    // heads*koff + h*n_k[i]; sequences without queries get no descriptor
    int ns = 0;
    long long qoff = 0, koff = 0;
    for (int i = 0; i < n_seqs; ++i) {
        if (n_q[i] > 0) {
            AttnStreamDesc& a = p.st[ns++];
            a.n_q = n_q[i];
            a.n_k = n_k[i];
            a.q_row0 = (int)(heads * qoff);
            a.kv_row0 = (int)(heads * koff);
            a.kv_head_stride = n_k[i];
            a.out_tok0 = (int)qoff;
        }
        qoff += n_q[i];
        koff += n_k[i];
    }
    p.n_streams = ns;
    if (plan_attention(p, n_sm, n_part, (int)n_cnt) < 0)
        return fail(PV_ERR_CAPACITY, "attention plan exceeds the workspace");
    CUtensorMap tq, tk, tv;
    char msg[256];
    CUtensorMap to;
    if (!encode_rows_map(&tq, q, heads * tot_q, head_dim, msg, sizeof msg) ||
        !encode_rows_map(&tk, k, heads * tot_k, head_dim, msg, sizeof msg) ||
        !encode_rows_map(&tv, v, heads * tot_k, head_dim, msg, sizeof msg) ||
        !encode_out_map(&to, out, tot_q, heads, head_dim, msg, sizeof msg))
        return fail(PV_ERR_CUDA, "%s", msg);
    cudaError_t e = launch_attn(tq, tk, tv, to, p, (cudaStream_t)cuda_stream);
    if (e != cudaSuccess) return cuda_fail(e, "attn_varlen launch");
    return PV_OK;
}

pv_status pv_attn_plan(int n_seqs, const int* n_q, const int* n_k, int heads, int n_sm,
                       int partial_slots, int* grid, int* mode, long long* ranges) {
    if (!grid || !mode || !ranges) return fail(PV_ERR_INVALID_ARG, "NULL output pointer");
    long long tot_q = 0, tot_k = 0;
    size_t n_cnt = 0, tiles = 0;
    pv_status st = varlen_sizes(n_seqs, n_q, n_k, heads, 128, &tot_q, &tot_k, &n_cnt, &tiles);
    if (st) return st;
    if (tot_q == 0) return fail(PV_ERR_SHAPE, "no queries");
    if (n_sm < 1 || partial_slots < 0) return fail(PV_ERR_INVALID_ARG, "n_sm < 1 or slots < 0");
    AttnParams p{};
    p.heads = heads;
    int ns = 0;
    for (int i = 0; i < n_seqs; ++i) {
        if (n_q[i] == 0) continue;
        p.st[ns].n_q = n_q[i];
        p.st[ns].n_k = n_k[i];
        ++ns;
    }
    p.n_streams = ns;
    if (plan_attention(p, n_sm, partial_slots, (int)n_cnt) < 0)
        return fail(PV_ERR_CAPACITY, "no plan fits");
    *grid = p.grid;
    *mode = p.item_aligned;
    // stream-K: the key-tile range of every CTA, as the kernel derives it;
    // whole items at run time: no fixed ranges, only the two ends
    for (int c = 0; c <= p.grid; ++c)
        ranges[c] = p.item_aligned == 0 ? (long long)c * p.total / p.grid
                                        : (c == 0 ? 0 : c == p.grid ? p.total : -1);
    return PV_OK;
}

pv_status pv_euler_step(float* x, const float* v, size_t n, float dsigma, void* cuda_stream) {
    if (n == 0) return PV_OK;
    if (!x || !v) return fail(PV_ERR_INVALID_ARG, "NULL tensor pointer");
    if (!aligned(x, 4) || !aligned(v, 4)) return fail(PV_ERR_INVALID_ARG, "misaligned f32 tensor");
    if (!std::isfinite(dsigma)) return fail(PV_ERR_INVALID_ARG, "dsigma is not finite");
    pv_status st;
    if ((st = check_async("an earlier launch"))) return st;
    cudaError_t e = launch_euler(x, v, n, dsigma, (cudaStream_t)cuda_stream);
    if (e != cudaSuccess) return cuda_fail(e, "euler launch");
    return PV_OK;
}

pv_status pv_sigma_schedule(int n_steps, double shift, double sigma_max, double* sigmas_out,
                            int* timesteps_out) {
    if (n_steps < 1 || !sigmas_out) return fail(PV_ERR_INVALID_ARG, "n_steps < 1 or NULL output");
    if (!(shift > 0.0) || !std::isfinite(shift)) return fail(PV_ERR_INVALID_ARG, "shift must be > 0");
    if (sigma_max <= 0.0) sigma_max = 1.0 - 1.0 / 1000.0;
    if (!(sigma_max <= 1.0)) return fail(PV_ERR_INVALID_ARG, "sigma_max must be in (0, 1]");
    for (int i = 0; i < n_steps; ++i) {
        const double u = sigma_max * (1.0 - (double)i / n_steps);
        sigmas_out[i] = shift * u / (1.0 + (shift - 1.0) * u);
        if (timesteps_out) timesteps_out[i] = (int)std::floor(1000.0 * sigmas_out[i]);
    }
    sigmas_out[n_steps] = 0.0;
    return PV_OK;
}

pv_status pv_euler_cfg_step(float* x, const float* v_cond, const float* v_uncond, size_t n,
                            float guide_scale, float dsigma, void* cuda_stream) {
    if (n == 0) return PV_OK;
    if (!x || !v_cond || !v_uncond) return fail(PV_ERR_INVALID_ARG, "NULL tensor pointer");
    if (!aligned(x, 4) || !aligned(v_cond, 4) || !aligned(v_uncond, 4))
        return fail(PV_ERR_INVALID_ARG, "misaligned f32 tensor");
    if (!std::isfinite(dsigma) || !std::isfinite(guide_scale))
        return fail(PV_ERR_INVALID_ARG, "dsigma and guide_scale must be finite");
    pv_status st;
    if ((st = check_async("an earlier launch"))) return st;
    cudaError_t e = launch_euler_cfg(x, v_cond, v_uncond, n, guide_scale, dsigma,
                                     (cudaStream_t)cuda_stream);
    if (e != cudaSuccess) return cuda_fail(e, "euler_cfg launch");
    return PV_OK;
}

pv_status pv_x0_estimate(float* x0, const float* x, const float* v, size_t n, float sigma,
                         void* cuda_stream) {
    if (n == 0) return PV_OK;
    if (!x0 || !x || !v) return fail(PV_ERR_INVALID_ARG, "NULL tensor pointer");
    if (!aligned(x0, 4) || !aligned(x, 4) || !aligned(v, 4))
        return fail(PV_ERR_INVALID_ARG, "misaligned f32 tensor");
    if (!std::isfinite(sigma)) return fail(PV_ERR_INVALID_ARG, "sigma must be finite");
    pv_status st;
    if ((st = check_async("an earlier launch"))) return st;
    cudaError_t e = launch_x0(x0, x, v, n, sigma, (cudaStream_t)cuda_stream);
    if (e != cudaSuccess) return cuda_fail(e, "x0 launch");
    return PV_OK;
}

pv_status pv_kv_poll_device_error(pv_kv kv, int* code) {
    if (!kv || !code) return fail(PV_ERR_INVALID_ARG, "NULL argument");
    *code = 0;
    if (!kv->device) return PV_OK;
    cudaError_t e = cudaMemcpy(code, kv->ws + kv->wl.err_off, sizeof(int), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, "reading the device error word");
    if (*code) {
        // an aborted launch may leave split-merge arrival counters part
        // counted: clear them with the error word
        e = cudaMemset(kv->ws + kv->wl.err_off, 0, sizeof(int));
        if (e == cudaSuccess)
            e = cudaMemset(kv->ws + kv->wl.cnt_off, 0, sizeof(int) * (size_t)kv->wl.n_counters);
        if (e != cudaSuccess) return cuda_fail(e, "clearing the device error word");
        return fail(PV_ERR_TIMEOUT, "a device-side wait gave up (code %d)", *code);
    }
    return PV_OK;
}

// The device error word of an attention workspace (ws), or of the fixed
// scratch of pv_attn_dense_noalloc (ws == NULL), and the bytes to re-zero
// after a timeout: the whole workspace (its arrival counters may be left part
// counted), or only the scratch's error block (each no-alloc call clears the
// counters it uses).
static pv_status attn_err_word(void* ws, size_t ws_bytes, char** base, size_t* clear) {
    if (ws) {
        if (!aligned(ws, 256) || ws_bytes < 256)
            return fail(PV_ERR_INVALID_ARG, "workspace %p of %zu bytes: need >= 256, 256-byte aligned",
                        ws, ws_bytes);
        *base = (char*)ws;
        *clear = ws_bytes;
        return PV_OK;
    }
    void* p = nullptr;
    cudaError_t e = noalloc_scratch_address(&p);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress of the no-alloc scratch");
    *base = (char*)p;
    *clear = 256;
    return PV_OK;
}

pv_status pv_attn_poll_device_error(void* ws, size_t ws_bytes, int* code, void* cuda_stream) {
    if (!code) return fail(PV_ERR_INVALID_ARG, "NULL argument");
    *code = 0;
    char* base = nullptr;
    size_t clear = 0;
    pv_status st = attn_err_word(ws, ws_bytes, &base, &clear);
    if (st) return st;
    cudaError_t e = cudaStreamSynchronize((cudaStream_t)cuda_stream);
    if (e == cudaSuccess) e = cudaMemcpy(code, base, sizeof(int), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, "reading the device error word");
    if (*code) {
        e = cudaMemset(base, 0, clear);
        if (e != cudaSuccess) return cuda_fail(e, "clearing the device error word");
        return fail(PV_ERR_TIMEOUT, "a device-side wait gave up (code %d)", *code);
    }
    return PV_OK;
}

pv_status pv_attn_selftest_wait_timeout(void* ws, void* cuda_stream) {
    char* base = nullptr;
    size_t clear = 0;
    pv_status st = attn_err_word(ws, ws ? 256 : 0, &base, &clear);
    if (st) return st;
    if ((st = check_async("an earlier launch"))) return st;
    cudaError_t e = launch_wait_timeout_probe((int*)base, (cudaStream_t)cuda_stream);
    if (e != cudaSuccess) return cuda_fail(e, "wait-timeout self-test launch");
    return PV_OK;
}

pv_status pv_kv_selftest_wait_timeout(pv_kv kv, void* cuda_stream) {
    if (!kv) return fail(PV_ERR_INVALID_ARG, "handle is NULL");
    if (!kv->device) return fail(PV_ERR_STATE, "bookkeeping-only handle has no device buffers");
    pv_status st;
    if ((st = check_async("an earlier launch"))) return st;
    cudaError_t e = launch_wait_timeout_probe((int*)(kv->ws + kv->wl.err_off),
                                              (cudaStream_t)cuda_stream);
    if (e != cudaSuccess) return cuda_fail(e, "wait-timeout self-test launch");
    return PV_OK;
}

}  // extern "C"
