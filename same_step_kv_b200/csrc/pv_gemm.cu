// The q, k, v projection of the tokens as one tcgen05 GEMM, with the first
// half of the QK-Norm in its epilogue.
//
// y[t][n] = sum_c x[t][c] * w[n][c] + b[n] for the tokens t of a launch and
// the 3 * dim output features n (q, then k, then v; w stored [out][in] as a
// linear layer keeps it), kept in f32, and for each token the sums of squares
// of its q features and of its k features, ss[t][0] and ss[t][1].  The second
// half of the norm (scale by rsqrt(ss / dim + eps) and the gain) runs where y
// is read next, in the RoPE / append kernel.  Blog "Learning Video Generation
// from the Wan2.2 Source Code", chapter 4, end of "3D RoPE": q and k pass
// through their linear layers, then an RMSNorm.
//
// One CTA computes a 256-token x BN-feature tile as two 128-token halves that
// share each slice of w in shared memory (half the w traffic per FLOP of a
// 128-token tile; for the 880 x 3072 chunk the 4 x 36 tiles are one wave on
// 148 SMs).  Warp 0 loads 64-column slices of x and w with TMA into a ring
// of stages (128-byte swizzle); warp 1 runs the issue loop with all lanes and
// one elected lane issues the tcgen05.mma (M = 128, N = BN, K = 16, one f32
// accumulator per half in TMEM); then all 8 warps (two per TMEM lane
// quadrant, one per half, one token per thread) add the bias, sum the squares
// and stage the tile in the freed ring for TMA stores.  A half beyond the last token is
// neither loaded nor multiplied.  Every wait on an mbarrier is bounded.
//
// kFused: the whole QK-Norm, RoPE and append in the epilogue, for a launch
// whose tiles are all resident at once (a cooperative launch of at most one
// CTA per SM).  The RMSNorm's factor of a token needs the sums of squares of
// all dim / BN feature tiles of its q (or k), which other CTAs compute: each
// CTA writes its tile's partial sums to its own slots, then sets its flag to
// the call's epoch, and waits (bounded) until the flags of all tiles of its
// token block hold the epoch; it adds the partial sums in tile order (the
// same result whatever the timing), forms the factor, applies it with the
// gain and the rotation to its tile,
// still in TMEM, and writes bf16 q_rot and the K/V rows of the store.  v gets
// the bias only.  No f32 y is written.  While the MMAs run, warps 2-7 stage
// the tile's bias and gain and (when it fits) the whole RoPE cos / sin table
// in shared memory beside the ring (the fused launch is only taken when it
// fits), so the epilogue's per-token lookups stay on chip.  Each warp stages
// its 32 tokens' bf16 output in the freed ring as 32-row x 64-feature boxes
// in TMA's 128-byte swizzle and, when its tokens are 32 consecutive rows of
// one stream, stores each box with a TMA tensor store as soon as it is
// staged (q_rot, or the K / V rows of every destination); otherwise (the
// ragged last rows, a warp across two streams) its lanes write the rows.
#include "pv_internal.h"

namespace pv {
namespace {

constexpr int kGThreads = 256;
constexpr int kGM = 128;      // tokens per half tile (one MMA's M)
constexpr int kGHalves = 2;   // halves per tile
constexpr int kGK = 64;       // input features per stage (one 128-byte swizzle row of bf16)
constexpr int kGMaxStages = 4;
constexpr long long kGWait = 2000000000LL;  // ~1 s of clock64

template <int BN>
struct GCfg {
    static constexpr int kABytes = kGM * kGK * 2;          // one half's x slice
    static constexpr int kBBytes = BN * kGK * 2;
    static constexpr int kStageBytes = kGHalves * kABytes + kBBytes;
    static constexpr int kStages = BN == 256 ? 3 : kGMaxStages;
    static constexpr int kBarOff = kStages * kStageBytes;
    static constexpr int kSmem = kBarOff + 256 + 1024;
    // the epilogue stages 8 warps x 32 tokens x kEpiCols f32 per round in the freed ring
    static constexpr int kEpiCols = BN < 128 ? BN : 128;
    static_assert(8 * 32 * kEpiCols * 4 <= kBarOff, "epilogue staging does not fit the ring");
    static_assert(kBarOff + 256 + 1024 <= 227 * 1024, "shared memory");
};

struct GBars {
    uint64_t full[kGMaxStages];   // the stage's x and w slices have landed
    uint64_t empty[kGMaxStages];  // the MMAs reading the stage are done
    uint64_t done;             // every MMA of the tile is done
    uint32_t tmem;
    int abort;
};

__device__ __forceinline__ uint32_t g_smem(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void g_mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void g_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ bool g_try(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
// Bounded wait: false after ~1 s (the error word is set and the CTA aborts)
// or once another role of the CTA has aborted.
__device__ __forceinline__ bool g_wait(uint32_t bar, uint32_t parity, GBars* b, int* err) {
    if (g_try(bar, parity)) return true;
    const long long t0 = clock64();
    while (!g_try(bar, parity)) {
        if (*(volatile int*)&b->abort) return false;
        if (clock64() - t0 > kGWait) {
            atomicExch(err, 1);
            *(volatile int*)&b->abort = 1;
            return false;
        }
    }
    return true;
}
__device__ __forceinline__ void g_tma_load(uint32_t dst, const CUtensorMap* map, int x, int y,
                                           uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}
__device__ __forceinline__ void g_tma_store(const CUtensorMap* map, uint32_t src, int x, int y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
            reinterpret_cast<uint64_t>(map)),
        "r"(x), "r"(y), "r"(src)
        : "memory");
}
__device__ __forceinline__ void g_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void g_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// issued by the lane that elect.sync picks; the whole warp executes it
__device__ __forceinline__ void g_commit(uint32_t bar) {
    asm volatile(
        "{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
        "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(
            bar)
        : "memory");
}
__device__ __forceinline__ void g_mma(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc,
                                      uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred e, p;\n\telect.sync _|e, 0xffffffff;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
        "l"(a), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}
// shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups
// 1024 bytes apart (version 1)
__device__ __forceinline__ uint64_t g_desc(uint32_t addr) {
    return (uint64_t)((addr >> 4) & 0x3FFF) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
           (1ull << 46) | (2ull << 61);
}
// kind::f16 instruction descriptor: bf16 A and B (K-major), f32 D, M x N
__host__ __device__ constexpr uint32_t g_idesc(int M, int N) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(M >> 4) << 24);
}
__device__ __forceinline__ void g_tmem_ld32(uint32_t taddr, uint32_t* r) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
          "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
          "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
}

// 64 consecutive columns of this warp's 32 TMEM lanes, one load and its wait
__device__ __forceinline__ void g_tmem_ld64(uint32_t taddr, uint32_t* r) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x64.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%64];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]), "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
        : "r"(taddr)
        : "memory");
}

__device__ __forceinline__ uint32_t g_pack(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

template <int BN, bool kFused>
__global__ void __launch_bounds__(kGThreads, 1)
    qkv_gemm_kernel(const __grid_constant__ CUtensorMap tx, const __grid_constant__ CUtensorMap tw,
                    const __grid_constant__ CUtensorMap ty, const float* __restrict__ bias,
                    float* __restrict__ ss, int tokens, int dim, int* err,
                    const __grid_constant__ RopeParams rp, unsigned long long* flags,
                    unsigned long long epoch,
                    const __grid_constant__ QkvOutMaps om) {
    using C = GCfg<BN>;
    extern __shared__ __align__(1024) uint8_t g_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(g_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    GBars* b = reinterpret_cast<GBars*>(smem + C::kBarOff);
    const int warp = threadIdx.x / 32;
    const int lane = threadIdx.x & 31;
    constexpr int kStages = C::kStages;
    const int m0 = blockIdx.x * (kGM * kGHalves);
    const int n0 = blockIdx.y * BN;
    const int nk = dim / kGK;
    const int halves = m0 + kGM < tokens ? 2 : 1;  // the second half holds tokens
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            g_mbar_init(g_smem(&b->full[s]), 1);
            g_mbar_init(g_smem(&b->empty[s]), 1);
        }
        g_mbar_init(g_smem(&b->done), 1);
        b->abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         g_smem(&b->tmem)),
                     "r"((uint32_t)(kGHalves * BN))
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    g_fence_before();
    __syncthreads();
    g_fence_after();
    const uint32_t tmem = b->tmem;
    if (warp == 0) {
        if (lane == 0) {
            // producer: x rows m0.. (one or two halves), w rows n0.., 64 input
            // features per stage
            int issued = 0;
            for (int kb = 0; kb < nk; ++kb) {
                const int s = kb % kStages;
                if (kb >= kStages && !g_wait(g_smem(&b->empty[s]), ((kb / kStages) - 1) & 1, b, err))
                    break;
                const uint32_t full = g_smem(&b->full[s]);
                g_expect_tx(full, halves * C::kABytes + C::kBBytes);
                const uint32_t st = g_smem(smem + s * C::kStageBytes);
                for (int u = 0; u < halves; ++u)
                    g_tma_load(st + u * C::kABytes, &tx, kb * kGK, m0 + u * kGM, full);
                g_tma_load(st + kGHalves * C::kABytes, &tw, kb * kGK, n0, full);
                ++issued;
            }
            // no copy of ours may still be landing when the CTA leaves
            for (int i = issued > kStages ? issued - kStages : 0; i < issued; ++i) {
                const long long t0 = clock64();
                while (!g_try(g_smem(&b->full[i % kStages]), (i / kStages) & 1) &&
                       clock64() - t0 < kGWait) {
                }
            }
        }
    } else if (warp == 1) {
        // MMA issue: the whole warp runs the loop, one elected lane issues
        constexpr uint32_t idesc = g_idesc(kGM, BN);
        for (int kb = 0; kb < nk; ++kb) {
            const int s = kb % kStages;
            if (!__all_sync(0xffffffffu,
                            g_wait(g_smem(&b->full[s]), (kb / kStages) & 1, b, err)))
                break;
            g_fence_after();
            const uint32_t a = g_smem(smem + s * C::kStageBytes);
            const uint32_t bw = a + kGHalves * C::kABytes;
            for (int u = 0; u < halves; ++u) {
#pragma unroll
                for (int kk = 0; kk < kGK / 16; ++kk)
                    g_mma(tmem + u * BN, g_desc(a + u * C::kABytes + kk * 32), g_desc(bw + kk * 32),
                          idesc, (kb > 0 || kk > 0) ? 1u : 0u);
            }
            g_commit(g_smem(&b->empty[s]));  // the stage is free once these MMAs end
        }
        g_commit(g_smem(&b->done));
        // every MMA of ours has ended before TMEM is released
        const long long t0 = clock64();
        while (!g_try(g_smem(&b->done), 0) && clock64() - t0 < kGWait) {
        }
        __syncwarp();
    }
    // epilogue, all 8 warps: warp w reads TMEM lane quadrant w % 4 (one token
    // per thread) of half (w < 4 ? 1 : 0), so two warps share each SMSP
    if constexpr (kFused) {
        static_assert(8 * 32 * BN * 2 <= C::kBarOff, "output staging does not fit the ring");
        const int kind = n0 / dim;      // 0: q, 1: k, 2: v
        const int f0 = n0 - kind * dim;  // the tile's first feature within q, k or v
        float* sb = reinterpret_cast<float*>(smem + C::kBarOff + 256);
        float* sg = sb + BN;
        float2* stab = reinterpret_cast<float2*>(sg + BN);
        if (warp >= 2) {
            // while the MMAs run: bias, gain and the RoPE table into shared memory
            const float* gain = kind == 0 ? rp.g_q : rp.g_k;
            for (int i = threadIdx.x - 64; i < BN; i += kGThreads - 64) {
                sb[i] = __ldg(bias + n0 + i);
                sg[i] = kind < 2 ? __ldg(gain + f0 + i) : 0.f;
            }
            if (kind < 2) {
                const int n_tab = rp.tab_w0 + rp.frame_w * rp.pairs_w;
                for (int i = threadIdx.x - 64; i < n_tab; i += kGThreads - 64)
                    stab[i] = __ldg(rp.table + i);
            }
        }
        const int q4 = warp & 3;
        const int u = warp < 4 ? 1 : 0;
        const bool ok = __all_sync(0xffffffffu, g_wait(g_smem(&b->done), 0, b, err));
        __syncthreads();  // the staged bias, gain and table are visible
        const int t = m0 + u * kGM + q4 * 32 + lane;
        const uint32_t trow = tmem + ((uint32_t)(q4 * 32) << 16) + u * BN;
        const bool live = ok && u < halves;
        if (live) g_fence_after();
        float factor = 1.f;
        if (kind < 2) {
            // this tile's share of each token's sum of squares, to its own
            // slot: ss[t][kind][tile]
            const int nt = dim / BN;
            float* ssk = ss + (size_t)kind * nt + f0 / BN;
            if (live) {
                float sq = 0.f;
#pragma unroll 1
                for (int c = 0; c < BN; c += 64) {
                    uint32_t o[64];
                    g_tmem_ld64(trow + c, o);
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const float4 bj = *reinterpret_cast<const float4*>(sb + c + 4 * j);
                        const float a0 = __uint_as_float(o[4 * j + 0]) + bj.x;
                        const float a1 = __uint_as_float(o[4 * j + 1]) + bj.y;
                        const float a2 = __uint_as_float(o[4 * j + 2]) + bj.z;
                        const float a3 = __uint_as_float(o[4 * j + 3]) + bj.w;
                        sq = fmaf(a0, a0, fmaf(a1, a1, fmaf(a2, a2, fmaf(a3, a3, sq))));
                    }
                }
                if (t < tokens) ssk[(size_t)t * 2 * nt] = sq;
            }
            __syncthreads();
            // publish (the fence after the barrier releases every thread's
            // sums), then thread j < nt waits for tile j of the token block.
            // A CTA that gave up a wait publishes too: its sums are missing,
            // but the error word is set and the call's outputs are invalid
            // either way, and the other CTAs then end without waiting a second
            const unsigned cta = blockIdx.y * gridDim.x + blockIdx.x;
            if (threadIdx.x == 0) {
                asm volatile("fence.acq_rel.gpu;" ::: "memory");
                asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(flags + cta), "l"(epoch)
                             : "memory");
            }
            if (threadIdx.x < nt) {
                const unsigned long long* f = flags + (kind * nt + threadIdx.x) * gridDim.x + blockIdx.x;
                const long long w0 = clock64();
                for (;;) {
                    unsigned long long v;
                    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(f) : "memory");
                    if (v == epoch) break;
                    if (*(volatile int*)&b->abort) break;
                    if (clock64() - w0 > kGWait) {
                        atomicExch(err, 1);
                        *(volatile int*)&b->abort = 1;
                        break;
                    }
                }
            }
            __syncthreads();
            if (live && t < tokens && !*(volatile int*)&b->abort) {
                // all loads in flight at once, added in tile order
                const float* st = ss + (size_t)t * 2 * nt + (size_t)kind * nt;
                float part[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) part[j] = j < nt ? __ldcg(st + j) : 0.f;
                float sum = 0.f;
#pragma unroll
                for (int j = 0; j < 16; ++j) sum += part[j];
                for (int j = 16; j < nt; ++j) sum += __ldcg(st + j);
                factor = rsqrtf(sum / dim + rp.eps);
            }
        }
        // tcgen05.ld is a warp-wide instruction: the whole warp loads when
        // any of it goes on, and only the lanes that hold a token write
        if (__all_sync(0xffffffffu, live && !*(volatile int*)&b->abort)) {
            const bool row = t < tokens;
            const int tt = row ? t : tokens - 1;
            // the token's stream and position
            int si = 0;
            while (si + 1 < rp.n_streams && rp.st[si + 1].in_tok0 <= tt) ++si;
            const RopeStreamDesc& sd = rp.st[si];
            const int T = rp.frame_w * rp.frame_h;
            const int D = rp.head_dim;
            const int tl = tt - sd.in_tok0;
            const int fr = sd.frame0 + tl / T;
            const int r = tl % T;
            const int hh = r / rp.frame_w;
            const int ww = r - hh * rp.frame_w;
            const int it = fr * rp.pairs_t, ih = rp.tab_h0 + hh * rp.pairs_h - rp.pairs_t,
                      iw = rp.tab_w0 + ww * rp.pairs_w - rp.pairs_t - rp.pairs_h;
            // this warp's 32 rows of BN bf16 in the freed ring: BN / 64 boxes
            // of 32 rows x 128 bytes, 16-byte piece q of row r at
            // (q ^ (r & 7)) * 16 (TMA's 128-byte swizzle; no bank conflicts
            // for a row per lane, nor for 8 lanes per row)
            uint8_t* stg = smem + warp * (32 * BN * 2);
            // one TMA store per box when the 32 tokens are consecutive rows
            // of one stream
            // (every lane takes part in the shuffle: no short-circuit around it)
            const int si0 = __shfl_sync(0xffffffffu, si, 0);
            const bool bulk = __all_sync(0xffffffffu, row && si == si0);
            const CUtensorMap* omap = kind == 0 ? &om.q : kind == 1 ? &om.k : &om.v;
#pragma unroll 1
            for (int c = 0; c < BN; c += 64) {
                uint32_t o[64];
                g_tmem_ld64(trow + c, o);
                float y[64];
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const float4 bj = *reinterpret_cast<const float4*>(sb + c + 4 * j);
                    y[4 * j + 0] = __uint_as_float(o[4 * j + 0]) + bj.x;
                    y[4 * j + 1] = __uint_as_float(o[4 * j + 1]) + bj.y;
                    y[4 * j + 2] = __uint_as_float(o[4 * j + 2]) + bj.z;
                    y[4 * j + 3] = __uint_as_float(o[4 * j + 3]) + bj.w;
                }
                uint32_t w[32];
                if (kind < 2) {
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const float4 gj = *reinterpret_cast<const float4*>(sg + c + 4 * j);
                        y[4 * j + 0] *= factor * gj.x;
                        y[4 * j + 1] *= factor * gj.y;
                        y[4 * j + 2] *= factor * gj.z;
                        y[4 * j + 3] *= factor * gj.w;
                    }
                    // 64 columns lie in one head (D is 64 or 128)
                    const int pair0 = ((f0 + c) % D) / 2;
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const int pair = pair0 + i;
                        const int idx = pair < rp.pairs_t                 ? it + pair
                                        : pair < rp.pairs_t + rp.pairs_h ? ih + pair
                                                                          : iw + pair;
                        const float2 cs = stab[idx];
                        const float ax = y[2 * i], ay = y[2 * i + 1];
                        w[i] = g_pack(fmaf(ax, cs.x, -ay * cs.y), fmaf(ax, cs.y, ay * cs.x));
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) w[i] = g_pack(y[2 * i], y[2 * i + 1]);
                }
                uint8_t* box = stg + (c / 64) * 4096;
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    *reinterpret_cast<uint4*>(box + lane * 128 + ((q ^ (lane & 7)) << 4)) =
                        make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
                if (bulk) {
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    __syncwarp();
                    if (lane == 0) {
                        // lane 0 holds the warp's first token
                        const int h = (f0 + c) / D;
                        const int d0 = (f0 + c) - h * D;
                        if (kind == 0) {
                            g_tma_store(omap, g_smem(box), d0,
                                        (int)(sd.qrot_row0 + (long long)h * sd.n_tok + tl));
                        } else {
                            for (int dd = 0; dd < sd.n_dst; ++dd)
                                g_tma_store(omap, g_smem(box), d0,
                                            (int)(sd.dst_row0[dd] + h * rp.dst_head_stride + tl));
                        }
                        asm volatile("cp.async.bulk.commit_group;" ::: "memory");
                    }
                }
            }
            if (bulk) {
                // the stores have finished before the CTA leaves
                if (lane == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
                __syncwarp();
            } else {
                __syncwarp();
                // per head segment of L = min(BN, D) features, each token's L
                // bf16 are contiguous in q_rot or the K / V rows; lpr lanes
                // write one token's segment, 32 / lpr tokens per instruction
                const int L = BN < D ? BN : D;
                const int lpr = L / 8;
                const int pc = lane % lpr;
                const int rsub = lane / lpr;
                bf16* dbase = kind == 0 ? rp.q_rot : kind == 1 ? rp.k_dst : rp.v_dst;
                const long long hstride = kind == 0 ? (long long)sd.n_tok : rp.dst_head_stride;
                const int nd = kind == 0 ? 1 : __reduce_max_sync(0xffffffffu, sd.n_dst);
                for (int dd = 0; dd < nd; ++dd) {
                    // row of head 0 for this lane's token, -1 for none
                    long long mine = -1;
                    if (row) {
                        if (kind == 0)
                            mine = sd.qrot_row0 + tl;
                        else if (dd < sd.n_dst)
                            mine = sd.dst_row0[dd] + tl;
                    }
                    for (int sg0 = 0; sg0 < BN; sg0 += L) {
                        const int h = (f0 + sg0) / D;
                        const int d0 = (f0 + sg0) - h * D;
                        // this lane's token segment in the output, NULL for none
                        bf16* const own = mine >= 0 ? dbase + (mine + h * hstride) * D + d0 : nullptr;
#pragma unroll 4
                        for (int i = 0; i < 32; i += 32 / lpr) {
                            const int rr = i + rsub;
                            bf16* const dst = reinterpret_cast<bf16*>(
                                __shfl_sync(0xffffffffu, reinterpret_cast<unsigned long long>(own), rr));
                            const int pp = sg0 / 8 + pc;  // 16-byte piece of the staged row
                            const uint4 val = *reinterpret_cast<const uint4*>(
                                stg + (pp / 8) * 4096 + rr * 128 + (((pp & 7) ^ (rr & 7)) << 4));
                            if (dst) *reinterpret_cast<uint4*>(dst + pc * 8) = val;
                        }
                    }
                }
            }
        }
    } else {
        const int q4 = warp & 3;
        const int u = warp < 4 ? 1 : 0;
        const bool ok = __all_sync(0xffffffffu, g_wait(g_smem(&b->done), 0, b, err));
        if (ok && u < halves && !*(volatile int*)&b->abort) {
            g_fence_after();
            const int kind = n0 / dim;  // 0: q, 1: k, 2: v
            constexpr int kCols = C::kEpiCols;  // columns staged per round
            // 32 tokens x kCols f32 of this warp, in 32-column boxes of 4 KB,
            // staged in the ring that the MMAs no longer read
            uint8_t* buf = smem + warp * (32 * kCols * 4);
            const int row0 = m0 + u * kGM + q4 * 32;  // this warp's first token
            const int grow = row0 + lane;
            float sq = 0.f;
            for (int c0 = 0; c0 < BN; c0 += kCols) {
                if (c0 > 0) {
                    // the previous round's stores have read the staging buffer
                    if (lane == 0) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
                    __syncwarp();
                }
#pragma unroll 1
                for (int c = c0; c < c0 + kCols; c += 32) {
                    uint32_t o[32];
                    g_tmem_ld32(tmem + ((uint32_t)(q4 * 32) << 16) + u * BN + c, o);
                    uint8_t* box = buf + ((c - c0) / 32) * 4096;
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const float4 bj = __ldg(reinterpret_cast<const float4*>(bias + n0 + c + 4 * j));
                        float4 v;
                        v.x = __uint_as_float(o[4 * j + 0]) + bj.x;
                        v.y = __uint_as_float(o[4 * j + 1]) + bj.y;
                        v.z = __uint_as_float(o[4 * j + 2]) + bj.z;
                        v.w = __uint_as_float(o[4 * j + 3]) + bj.w;
                        sq = fmaf(v.x, v.x, fmaf(v.y, v.y, fmaf(v.z, v.z, fmaf(v.w, v.w, sq))));
                        // 16-byte chunk j of row `lane`, 128-byte swizzle
                        *reinterpret_cast<float4*>(box + lane * 128 + ((j ^ (lane & 7)) << 4)) = v;
                    }
                }
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                __syncwarp();
                if (lane == 0 && row0 < tokens) {
                    for (int c = c0; c < c0 + kCols; c += 32)
                        g_tma_store(&ty, g_smem(buf + ((c - c0) / 32) * 4096), n0 + c, row0);
                    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
                }
            }
            if (kind < 2 && grow < tokens) atomicAdd(ss + (size_t)grow * 2 + kind, sq);
            if (lane == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
            __syncwarp();
        }
    }
    g_fence_before();
    __syncthreads();
    if (warp == 1) {
        g_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"((uint32_t)(kGHalves * BN))
                     : "memory");
    }
}

template <int BN>
cudaError_t launch_gemm_bn(const CUtensorMap& tx, const CUtensorMap& tw, const CUtensorMap& ty,
                           const float* bias, float* ss, int tokens, int dim, int* err,
                           cudaStream_t s) {
    using C = GCfg<BN>;
    static std::atomic<unsigned long long> configured{0};
    const cudaError_t e = smem_limit_once(qkv_gemm_kernel<BN, false>, C::kSmem, configured);
    if (e != cudaSuccess) return e;
    dim3 grid((tokens + kGM * kGHalves - 1) / (kGM * kGHalves), 3 * dim / BN);
    RopeParams none{};
    QkvOutMaps no_maps{};
    qkv_gemm_kernel<BN, false><<<grid, kGThreads, C::kSmem, s>>>(tx, tw, ty, bias, ss, tokens, dim,
                                                                 err, none, nullptr, 0ull, no_maps);
    return cudaGetLastError();
}

// One cooperative launch of the fused kernel, or cudaErrorCooperativeLaunchTooLarge
// when its tiles cannot all be resident at once (the caller then takes the
// two-launch path).
template <int BN>
cudaError_t launch_fused_bn(const CUtensorMap& tx, const CUtensorMap& tw, const float* bias,
                            float* ss, unsigned long long* flags, unsigned long long epoch,
                            int tokens, int dim, int* err, const RopeParams& rp,
                            const QkvOutMaps& om, cudaStream_t s) {
    using C = GCfg<BN>;
    constexpr int kMaxSmem = 227 * 1024;
    static std::atomic<unsigned long long> configured{0};
    cudaError_t e = smem_limit_once(qkv_gemm_kernel<BN, true>, kMaxSmem, configured);
    if (e != cudaSuccess) return e;
    // bias and gain of the tile, then the RoPE table, all beside the ring
    const long long n_tab = (long long)rp.tab_w0 + (long long)rp.frame_w * rp.pairs_w;
    if (C::kSmem + 2 * BN * 4 + n_tab * 8 > kMaxSmem) return cudaErrorCooperativeLaunchTooLarge;
    const int smem = C::kSmem + 2 * BN * 4 + (int)(n_tab * 8);
    const dim3 grid((tokens + kGM * kGHalves - 1) / (kGM * kGHalves), 3 * dim / BN);
    int dev = 0, n_sm = 0, per_sm = 0, coop = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev);
    cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev);
    if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, qkv_gemm_kernel<BN, true>,
                                                           kGThreads, smem)) != cudaSuccess)
        return e;
    if (!coop || (long long)grid.x * grid.y > (long long)per_sm * n_sm ||
        (long long)grid.x * grid.y > kQkvFlags || dim / BN > kGThreads)
        return cudaErrorCooperativeLaunchTooLarge;
    CUtensorMap ty = tx;  // not read by the fused epilogue
    void* args[] = {(void*)&tx, (void*)&tw, (void*)&ty, (void*)&bias, (void*)&ss,
                    (void*)&tokens, (void*)&dim, (void*)&err, (void*)&rp, (void*)&flags,
                    (void*)&epoch, (void*)&om};
    return cudaLaunchCooperativeKernel((const void*)qkv_gemm_kernel<BN, true>, grid,
                                       dim3(kGThreads), args, smem, s);
}

}  // namespace

int qkv_gemm_tile_n(int dim) {
    return dim % 256 == 0 ? 256 : dim % 128 == 0 ? 128 : dim % 64 == 0 ? 64 : 0;
}

cudaError_t launch_qkv_gemm(const CUtensorMap& tx, const CUtensorMap& tw, const CUtensorMap& ty,
                            const float* bias, float* ss, int tokens, int dim, int* err,
                            cudaStream_t s) {
    switch (qkv_gemm_tile_n(dim)) {
        case 256: return launch_gemm_bn<256>(tx, tw, ty, bias, ss, tokens, dim, err, s);
        case 128: return launch_gemm_bn<128>(tx, tw, ty, bias, ss, tokens, dim, err, s);
        case 64: return launch_gemm_bn<64>(tx, tw, ty, bias, ss, tokens, dim, err, s);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_qkv_fused(const CUtensorMap& tx, const CUtensorMap& tw, const float* bias,
                             float* ss, unsigned long long* flags, unsigned long long epoch,
                             int tokens, int dim, int* err, const RopeParams& rp,
                             const QkvOutMaps& om, cudaStream_t s) {
    switch (qkv_gemm_tile_n(dim)) {
        case 256:
            return launch_fused_bn<256>(tx, tw, bias, ss, flags, epoch, tokens, dim, err, rp, om, s);
        case 128:
            return launch_fused_bn<128>(tx, tw, bias, ss, flags, epoch, tokens, dim, err, rp, om, s);
        case 64:
            return launch_fused_bn<64>(tx, tw, bias, ss, flags, epoch, tokens, dim, err, rp, om, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace pv
