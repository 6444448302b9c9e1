// pv_attn_dense_noalloc: dense attention whose split-KV scratch lives in a
// fixed array inside this library instead of a caller-provided workspace.
//
// Some callers cannot allocate device memory at the point where they call
// us: code running inside a custom allocator or memory-pool callback (where
// allocating would re-enter the allocator), plugins whose host framework owns
// every device allocation and forbids its own, and latency-critical paths
// that must not take the allocator's locks or risk an out-of-memory failure
// in the middle of a stream of work.  For them this entry point needs nothing
// but the inputs and outputs, and calls no cudaMalloc, cudaFree or other
// allocating routine.
//
// The scratch is one file-scope device array of kScratchBytes (8 MiB) that
// every GPU loading this library holds until the process exits.  It holds an
// error word, the split-KV arrival counters (at most kMaxCounters query
// tiles) and as many partial-result slots as fit; when they do not suffice for
// one CTA per SM, the planner gives each CTA whole query blocks instead.
#include <cmath>
#include <cstdio>
#include <mutex>

#include "pv_internal.h"

namespace pv {
namespace {

constexpr size_t kScratchBytes = 8u << 20;
constexpr size_t kErrBytes = 256;
constexpr int kMaxCounters = 16384;  // 64 KiB of arrival counters
constexpr size_t kPartOff = kErrBytes + kMaxCounters * sizeof(int);

static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_addr[kMaxDevices] = {};

// Device address of g_scratch on the current device, looked up once per
// device with that device current.  In host code `g_scratch` names a
// host-side stand-in, not device memory; only this address may reach a kernel.
cudaError_t scratch_address(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_addr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_scratch);
        if (e != cudaSuccess) return e;
        g_addr[dev] = p;
    }
    *out = g_addr[dev];
    return cudaSuccess;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace

cudaError_t noalloc_scratch_address(void** out) { return scratch_address(out); }

}  // namespace pv

using namespace pv;

extern "C" pv_status pv_attn_dense_noalloc(const void* q, const void* k, const void* v, int n_q,
                                           int n_k, int heads, int head_dim, void* out,
                                           float* lse, void* cuda_stream) {
    char msg[320];
    if (!q || !k || !v || !out)
        return report_error(PV_ERR_INVALID_ARG, "pv_attn_dense_noalloc: NULL tensor pointer");
    if (n_q < 1 || n_k < 1 || heads < 1 || (head_dim != 64 && head_dim != 128))
        return report_error(PV_ERR_SHAPE, "pv_attn_dense_noalloc: n_q, n_k, heads must be "
                                          "positive and head_dim 64 or 128");
    if (n_q > (1 << 30) || n_k > (1 << 30))  // the rounded tile counts stay in int
        return report_error(PV_ERR_SHAPE, "pv_attn_dense_noalloc: n_q or n_k above 2^30");
    if ((long long)n_q * heads >= (1LL << 31) || (long long)n_k * heads >= (1LL << 31))
        return report_error(PV_ERR_SHAPE, "pv_attn_dense_noalloc: too many rows for a tensor map");
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out))
        return report_error(PV_ERR_INVALID_ARG,
                            "pv_attn_dense_noalloc: tensors must be 16-byte aligned");
    const long long n_qb = (n_q + kQBlock - 1) / kQBlock;
    const long long n_cnt = (long long)heads * n_qb * kQTilesPerCta;
    if (n_cnt > kMaxCounters) {
        snprintf(msg, sizeof msg,
                 "pv_attn_dense_noalloc: heads * ceil(n_q / 256) * 2 = %lld query tiles exceeds "
                 "the %d that its fixed %zu-byte scratch supports; use pv_attn_dense",
                 n_cnt, kMaxCounters, kScratchBytes);
        return report_error(PV_ERR_CAPACITY, msg);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
        snprintf(msg, sizeof msg, "an earlier launch: %s", cudaGetErrorString(e));
        return report_error(PV_ERR_CUDA, msg);
    }
    int dev = 0, n_sm = 148, major = 0, minor = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
    if (major != 10 || minor != 0) {
        snprintf(msg, sizeof msg, "device %d is sm_%d%d; libpv is built for sm_100a", dev, major,
                 minor);
        return report_error(PV_ERR_UNSUPPORTED_ARCH, msg);
    }
    void* base = nullptr;
    if ((e = scratch_address(&base)) != cudaSuccess) {
        snprintf(msg, sizeof msg, "pv_attn_dense_noalloc: cudaGetSymbolAddress: %s",
                 cudaGetErrorString(e));
        return report_error(PV_ERR_CUDA, msg);
    }
    char* s = static_cast<char*>(base);
    cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
    // The array keeps the previous call's contents: the error word and the
    // arrival counters that this call uses must start at zero.
    e = cudaMemsetAsync(s, 0, kErrBytes + (size_t)n_cnt * sizeof(int), st);
    if (e != cudaSuccess) {
        snprintf(msg, sizeof msg, "pv_attn_dense_noalloc: clearing the scratch: %s",
                 cudaGetErrorString(e));
        return report_error(PV_ERR_CUDA, msg);
    }
    const int n_part =
        (int)((kScratchBytes - kPartOff) / (partial_slot_floats(head_dim) * sizeof(float)));
    AttnParams p{};
    p.out = static_cast<bf16*>(out);
    p.lse = lse;
    p.err = reinterpret_cast<int*>(s);
    p.counters = reinterpret_cast<int*>(s + kErrBytes);
    p.partial = reinterpret_cast<float*>(s + kPartOff);
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
    if (plan_attention(p, n_sm, n_part, kMaxCounters) < 0)
        return report_error(PV_ERR_CAPACITY, "pv_attn_dense_noalloc: no plan fits the scratch");
    CUtensorMap tq, tk, tv, to;
    if (!encode_rows_map(&tq, q, (long long)heads * n_q, head_dim, msg, sizeof msg) ||
        !encode_rows_map(&tk, k, (long long)heads * n_k, head_dim, msg, sizeof msg) ||
        !encode_rows_map(&tv, v, (long long)heads * n_k, head_dim, msg, sizeof msg) ||
        !encode_out_map(&to, out, n_q, heads, head_dim, msg, sizeof msg))
        return report_error(PV_ERR_CUDA, msg);
    e = launch_attn(tq, tk, tv, to, p, st);
    if (e != cudaSuccess) {
        snprintf(msg, sizeof msg, "pv_attn_dense_noalloc launch: %s", cudaGetErrorString(e));
        return report_error(PV_ERR_CUDA, msg);
    }
    return PV_OK;
}
