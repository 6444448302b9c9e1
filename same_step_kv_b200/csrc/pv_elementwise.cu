// HBM-bound kernels: 3D RoPE + same-step KV append, and the Euler update.
#include "pv_internal.h"

namespace pv {
namespace {

__device__ __forceinline__ uint4 ld_stream(const bf16* p) {
    // read once: do not keep in L1
    return __ldcs(reinterpret_cast<const uint4*>(p));
}

__device__ __forceinline__ void st16(bf16* p, uint4 v) { *reinterpret_cast<uint4*>(p) = v; }

__device__ __forceinline__ float2 unpack(uint32_t w) {
    __nv_bfloat162 b = *reinterpret_cast<__nv_bfloat162*>(&w);
    return __bfloat1622float2(b);
}

__device__ __forceinline__ uint32_t pack(float lo, float hi) {
    __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&b);
}

// Blog "Learning Video Generation from the Wan2.2 Source Code", chapter 4,
// "3D RoPE": pair p of a head belongs to the time, height or width block and
// turns by that coordinate times the pair's frequency, as the complex product
// (x + i y) e^{i angle}.  One thread handles 8 consecutive dimensions (4
// pairs) of one (token, head) of q, k and v; rows are read and written with
// 128-bit coalesced accesses.
// kProj = false: q, k, v are bf16 [tokens][H][D].
// kProj = true: they are the f32 projection y [tokens][3 * dim] (pv_gemm.cu)
// and q, k get the rest of the QK-Norm first (same chapter): times
// rsqrt(ss / dim + eps), ss the token's sum of squares, then the gain.
template <bool kProj>
__global__ void __launch_bounds__(256) rope_append_kernel(const __grid_constant__ RopeParams p) {
    const RopeStreamDesc& sd = p.st[blockIdx.y];
    const int G = p.head_dim >> 3;                   // 16-byte groups per head row
    const int per_tok = p.heads * G;
    const int n_items = sd.n_tok * per_tok;
    const int T = p.frame_w * p.frame_h;
    for (int it = blockIdx.x * blockDim.x + threadIdx.x; it < n_items; it += gridDim.x * blockDim.x) {
        const int t = it / per_tok;
        const int j = it - t * per_tok;
        const int h = j / G;
        const int g = j - h * G;
        float qf[8], kf[8];
        uint4 vv;
        if (kProj) {
            const int dim = p.heads * p.head_dim;
            const int f0 = h * p.head_dim + g * 8;           // feature of this group
            const size_t row = (size_t)(sd.in_tok0 + t);
            const float* yq = p.y + row * 3 * dim + f0;
            const float sq = rsqrtf(__ldg(p.ss + row * 2) / dim + p.eps);
            const float sk = rsqrtf(__ldg(p.ss + row * 2 + 1) / dim + p.eps);
            const float4 q0 = __ldcs(reinterpret_cast<const float4*>(yq));
            const float4 q1 = __ldcs(reinterpret_cast<const float4*>(yq + 4));
            const float4 k0 = __ldcs(reinterpret_cast<const float4*>(yq + dim));
            const float4 k1 = __ldcs(reinterpret_cast<const float4*>(yq + dim + 4));
            const float4 v0 = __ldcs(reinterpret_cast<const float4*>(yq + 2 * dim));
            const float4 v1 = __ldcs(reinterpret_cast<const float4*>(yq + 2 * dim + 4));
            // the gains as four 16-byte loads (f0 is a multiple of 8)
            const float4 gq0 = __ldg(reinterpret_cast<const float4*>(p.g_q + f0));
            const float4 gq1 = __ldg(reinterpret_cast<const float4*>(p.g_q + f0 + 4));
            const float4 gk0 = __ldg(reinterpret_cast<const float4*>(p.g_k + f0));
            const float4 gk1 = __ldg(reinterpret_cast<const float4*>(p.g_k + f0 + 4));
            const float qa[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
            const float ka[8] = {k0.x, k0.y, k0.z, k0.w, k1.x, k1.y, k1.z, k1.w};
            const float gqa[8] = {gq0.x, gq0.y, gq0.z, gq0.w, gq1.x, gq1.y, gq1.z, gq1.w};
            const float gka[8] = {gk0.x, gk0.y, gk0.z, gk0.w, gk1.x, gk1.y, gk1.z, gk1.w};
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                qf[i] = qa[i] * sq * gqa[i];
                kf[i] = ka[i] * sk * gka[i];
            }
            vv = make_uint4(pack(v0.x, v0.y), pack(v0.z, v0.w), pack(v1.x, v1.y), pack(v1.z, v1.w));
        } else {
            const size_t in_off = ((size_t)(sd.in_tok0 + t) * p.heads + h) * p.head_dim + g * 8;
            const uint4 qv = ld_stream(p.q + in_off);
            const uint4 kv = ld_stream(p.k + in_off);
            vv = ld_stream(p.v + in_off);
            const uint32_t qw[4] = {qv.x, qv.y, qv.z, qv.w};
            const uint32_t kw[4] = {kv.x, kv.y, kv.z, kv.w};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const float2 a = unpack(qw[u]);
                const float2 b = unpack(kw[u]);
                qf[2 * u] = a.x;
                qf[2 * u + 1] = a.y;
                kf[2 * u] = b.x;
                kf[2 * u + 1] = b.y;
            }
        }
        const int f = sd.frame0 + t / T;
        const int r = t % T;
        const int hh = r / p.frame_w;
        const int ww = r - hh * p.frame_w;
        uint32_t qo[4], ko[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int pair = g * 4 + u;
            int idx;
            if (pair < p.pairs_t) {
                idx = f * p.pairs_t + pair;
            } else if (pair < p.pairs_t + p.pairs_h) {
                idx = p.tab_h0 + hh * p.pairs_h + (pair - p.pairs_t);
            } else {
                idx = p.tab_w0 + ww * p.pairs_w + (pair - p.pairs_t - p.pairs_h);
            }
            const float2 cs = __ldg(p.table + idx);
            const float ax = qf[2 * u], ay = qf[2 * u + 1];
            const float bx = kf[2 * u], by = kf[2 * u + 1];
            qo[u] = pack(fmaf(ax, cs.x, -ay * cs.y), fmaf(ax, cs.y, ay * cs.x));
            ko[u] = pack(fmaf(bx, cs.x, -by * cs.y), fmaf(bx, cs.y, by * cs.x));
        }
        const size_t qrow = (size_t)sd.qrot_row0 + (size_t)h * sd.n_tok + t;
        st16(p.q_rot + qrow * p.head_dim + g * 8, make_uint4(qo[0], qo[1], qo[2], qo[3]));
        const uint4 kout = make_uint4(ko[0], ko[1], ko[2], ko[3]);
        for (int d = 0; d < sd.n_dst; ++d) {
            const size_t row = (size_t)sd.dst_row0[d] + (size_t)h * p.dst_head_stride + t;
            st16(p.k_dst + row * p.head_dim + g * 8, kout);
            st16(p.v_dst + row * p.head_dim + g * 8, vv);
        }
    }
}

// Blog chapter 5 ("UniPC"): the first-order Euler step x <- x + dsigma * v
// with dsigma = sigma_next - sigma.  float4 path over the aligned body, a
// scalar path for the ragged head and tail.
__global__ void __launch_bounds__(256) euler_kernel(float* __restrict__ x,
                                                    const float* __restrict__ v, size_t n,
                                                    float dsigma) {
    const size_t stride = (size_t)gridDim.x * blockDim.x;
    const size_t tid = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    const bool vec = ((((uintptr_t)x) | ((uintptr_t)v)) & 15) == 0;
    if (vec) {
        const size_t n4 = n >> 2;
        float4* x4 = reinterpret_cast<float4*>(x);
        const float4* v4 = reinterpret_cast<const float4*>(v);
        for (size_t i = tid; i < n4; i += stride) {
            float4 a = x4[i];
            const float4 b = __ldcs(v4 + i);
            a.x = fmaf(dsigma, b.x, a.x);
            a.y = fmaf(dsigma, b.y, a.y);
            a.z = fmaf(dsigma, b.z, a.z);
            a.w = fmaf(dsigma, b.w, a.w);
            x4[i] = a;
        }
        for (size_t i = (n4 << 2) + tid; i < n; i += stride) x[i] = fmaf(dsigma, v[i], x[i]);
    } else {
        for (size_t i = tid; i < n; i += stride) x[i] = fmaf(dsigma, v[i], x[i]);
    }
}

// Euler step on the classifier-free-guided velocity (blog chapter 5, "CFG":
// uncond + w * (cond - uncond)), fused so that the guided velocity is never
// stored: x += dsigma * (vu + w * (vc - vu)).
__global__ void __launch_bounds__(256) euler_cfg_kernel(float* __restrict__ x,
                                                        const float* __restrict__ vc,
                                                        const float* __restrict__ vu, size_t n,
                                                        float w, float dsigma) {
    const size_t stride = (size_t)gridDim.x * blockDim.x;
    const size_t tid = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    const bool vec = ((((uintptr_t)x) | ((uintptr_t)vc) | ((uintptr_t)vu)) & 15) == 0;
    size_t done = 0;
    if (vec) {
        const size_t n4 = n >> 2;
        float4* x4 = reinterpret_cast<float4*>(x);
        const float4* c4 = reinterpret_cast<const float4*>(vc);
        const float4* u4 = reinterpret_cast<const float4*>(vu);
        for (size_t i = tid; i < n4; i += stride) {
            float4 a = x4[i];
            const float4 c = __ldcs(c4 + i), u = __ldcs(u4 + i);
            a.x = fmaf(dsigma, fmaf(w, c.x - u.x, u.x), a.x);
            a.y = fmaf(dsigma, fmaf(w, c.y - u.y, u.y), a.y);
            a.z = fmaf(dsigma, fmaf(w, c.z - u.z, u.z), a.z);
            a.w = fmaf(dsigma, fmaf(w, c.w - u.w, u.w), a.w);
            x4[i] = a;
        }
        done = n4 << 2;
    }
    for (size_t i = done + tid; i < n; i += stride)
        x[i] = fmaf(dsigma, fmaf(w, vc[i] - vu[i], vu[i]), x[i]);
}

// Clean-data estimate of flow matching (blog chapter 1): x0 = x - sigma * v.
__global__ void __launch_bounds__(256) x0_kernel(float* __restrict__ x0,
                                                 const float* __restrict__ x,
                                                 const float* __restrict__ v, size_t n,
                                                 float sigma) {
    const size_t stride = (size_t)gridDim.x * blockDim.x;
    const size_t tid = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    const bool vec = ((((uintptr_t)x0) | ((uintptr_t)x) | ((uintptr_t)v)) & 15) == 0;
    size_t done = 0;
    if (vec) {
        const size_t n4 = n >> 2;
        float4* o4 = reinterpret_cast<float4*>(x0);
        const float4* a4 = reinterpret_cast<const float4*>(x);
        const float4* v4 = reinterpret_cast<const float4*>(v);
        for (size_t i = tid; i < n4; i += stride) {
            const float4 a = __ldcs(a4 + i), b = __ldcs(v4 + i);
            o4[i] = make_float4(fmaf(-sigma, b.x, a.x), fmaf(-sigma, b.y, a.y),
                                fmaf(-sigma, b.z, a.z), fmaf(-sigma, b.w, a.w));
        }
        done = n4 << 2;
    }
    for (size_t i = done + tid; i < n; i += stride) x0[i] = fmaf(-sigma, v[i], x[i]);
}

// SMs of the current device, looked up once per device ordinal below 64.
int sm_count() {
    static std::atomic<int> cache[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) dev = 0;
    if (dev >= 0 && dev < 64) {
        const int c = cache[dev].load(std::memory_order_relaxed);
        if (c > 0) return c;
    }
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
        n = 148;
    if (dev >= 0 && dev < 64) cache[dev].store(n, std::memory_order_relaxed);
    return n;
}

}  // namespace

cudaError_t launch_rope(const RopeParams& p, int max_tok, cudaStream_t s) {
    const long long items = (long long)max_tok * p.heads * (p.head_dim / 8);
    if (items >= (1LL << 31)) return cudaErrorInvalidValue;
    // grid: enough CTAs per stream to cover the SMs a few times over
    const int per_stream = (int)std::min<long long>((items + 255) / 256,
                                                    std::max(1, 8 * sm_count() / p.n_streams));
    dim3 grid(per_stream, p.n_streams);
    if (p.y)
        rope_append_kernel<true><<<grid, 256, 0, s>>>(p);
    else
        rope_append_kernel<false><<<grid, 256, 0, s>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_euler_cfg(float* x, const float* vc, const float* vu, size_t n, float w,
                             float dsigma, cudaStream_t s) {
    const size_t want = (n / 4 + 255) / 256;
    const int grid = (int)std::max<size_t>(1, std::min<size_t>(want, (size_t)sm_count() * 8));
    euler_cfg_kernel<<<grid, 256, 0, s>>>(x, vc, vu, n, w, dsigma);
    return cudaGetLastError();
}

cudaError_t launch_x0(float* x0, const float* x, const float* v, size_t n, float sigma,
                      cudaStream_t s) {
    const size_t want = (n / 4 + 255) / 256;
    const int grid = (int)std::max<size_t>(1, std::min<size_t>(want, (size_t)sm_count() * 8));
    x0_kernel<<<grid, 256, 0, s>>>(x0, x, v, n, sigma);
    return cudaGetLastError();
}

cudaError_t launch_euler(float* x, const float* v, size_t n, float dsigma, cudaStream_t s) {
    const size_t want = (n / 4 + 255) / 256;
    const int grid = (int)std::max<size_t>(1, std::min<size_t>(want, (size_t)sm_count() * 8));
    euler_kernel<<<grid, 256, 0, s>>>(x, v, n, dsigma);
    return cudaGetLastError();
}

}  // namespace pv
