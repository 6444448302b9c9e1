// Chunk attention on the 5th-generation tensor cores (sm_100a).
//
// o[q] = sum_k softmax_k(q . k / sqrt(D)) v_k over a contiguous range of key
// rows, with the online softmax: the key range is walked in 128-key tiles,
// keeping per query row a running maximum m and sum l, and rescaling the
// output accumulator when m grows (PhysisServe Wan2.2-5B model card,
// "Inference profile": the chunk's same-step key set; blog "Learning Video
// Generation from the Wan2.2 Source Code", chapter 8: the two matrix
// products QK^T and PV).
//
// One CTA = 3 warpgroups (12 warps):
//   warp 0       TMA producer: the two Q tiles once, then K_j, V_j per key
//                tile into a ring of shared-memory stages (128-byte swizzle).
//   warp 1       allocates 512 TMEM columns and runs the MMA issue loop
//                with all lanes; one elected lane issues each tcgen05.mma:
//                S_X = Q_X K_j^T (SS form), O_X += P_X V_j (P from TMEM).
//   warps 2, 3   idle.  Warpgroup 0 gives registers to the other two.
//   warps 4..7   softmax of query tile A (TMEM lane = query row),
//   warps 8..11  softmax of query tile B.
// TMEM columns: S_A [0,128) S_B [128,256) O_A [256,256+D) O_B [256+D,256+2D);
// P_X (bf16 pairs) overwrites the first 64 columns of S_X.
// The MMA order PV_A(j-1), S_A(j), PV_B(j-1), S_B(j) lets tile B's softmax run
// while tile A's products are on the tensor pipe, and the other way round.
// Each P V is issued in two halves of 64 keys: the softmax hands over the
// first half of P as soon as it is stored and computes the second meanwhile.
// The running maximum is only moved when it grows by more than 8 (log2
// units), so O is rescaled rarely; P stays below 2^8 and the final
// normalisation uses the m that was actually applied, so the result is exact
// softmax up to rounding.
//
// Every mbarrier wait is bounded (about one second); a wait that gives up
// sets the device error word, makes the CTA skip its remaining work, waits
// (bounded) for its own copies and MMAs, frees TMEM and returns.
#include "pv_internal.h"

namespace pv {
namespace {

constexpr int kThreads = 384;
constexpr int kRegsLow = 96;    // warpgroup 0 after setmaxnreg.dec
constexpr int kRegsHigh = 200;  // softmax warpgroups after setmaxnreg.inc
static_assert(kRegsLow * 128 + 2 * kRegsHigh * 128 <= 168 * kThreads, "register split");
constexpr long long kWaitCycles = 2000000000LL;  // ~1 s at 1.9 GHz
constexpr int kRing = 4;  // slots of the run-time item hand-out

template <int D>
struct Cfg {
    static constexpr int kSub = D / 64;                      // 64-column swizzle sub-tiles
    static constexpr int kTileBytes = kQRows * D * 2;        // one 128-row tile
    static constexpr int kStages = D == 128 ? 4 : 8;         // K/V ring depth
    static constexpr int kQOff = 0;
    static constexpr int kKVOff = 2 * kTileBytes;
    // output staging: 32 rows x 64 columns of bf16 (4 KB) per softmax warp
    static constexpr int kEpiOff = kKVOff + kStages * kTileBytes;
    static constexpr int kEpiWarpBytes = kOutRows * 64 * 2;
    static constexpr int kBarOff = kEpiOff + 8 * kEpiWarpBytes;
    static constexpr int kSmem = kBarOff + 512 + 1024;       // + barriers + alignment slack
    static constexpr uint32_t kColsO = 256;
};

struct Bars {  // 344 bytes, inside the 512 reserved after the tiles
    uint64_t q_full;
    uint64_t q_empty;
    uint64_t o_empty[2];
    uint64_t ep_in[2];    // split epilogue: the 4 softmax warps of a tile wrote their partial
    uint64_t ep_out[2];   // split epilogue: the arrival count is in last[]
    uint64_t s_full[2];
    uint64_t p_full[2];
    uint64_t p_lo[2];     // [X]: the first 64 key columns of P are in TMEM
    uint64_t o_full[2];
    uint64_t mma_done;
    uint64_t kv_full[8];
    uint64_t rel[8];      // release events: the K/V tiles they free may be overwritten
    uint32_t tmem_base;
    int abort;
    int last[2];
    uint64_t ring_full[kRing];   // items handed out at run time (item_grab / item_take)
    uint64_t ring_empty[kRing];
    int ring[kRing];
};
static_assert(sizeof(Bars) <= 512, "barriers beyond their reserved bytes");

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

// ----------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
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

// Bounded wait: false when it gave up (the CTA is then aborting).
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, Bars* b, int* err) {
    if (mbar_try(bar, parity)) return true;
    const long long t0 = clock64();
    while (!mbar_try(bar, parity)) {
        if (*(volatile int*)&b->abort) return false;
        if (clock64() - t0 > kWaitCycles) {
            atomicExch(err, 1);
            *(volatile int*)&b->abort = 1;
            return false;
        }
    }
    return true;
}

// ----------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_load(uint32_t dst, const CUtensorMap* map, int x, int y,
                                         uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}

// TMA store of the box at (c0, c1, c2) of a 3D tensor map from shared memory,
// in this thread's bulk async-group.
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, uint32_t src, int c0, int c1,
                                             int c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%1, %2, %3}], [%4];" ::"l"(
            reinterpret_cast<uint64_t>(map)),
        "r"(c0), "r"(c1), "r"(c2), "r"(src)
        : "memory");
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// Wait until this thread's bulk stores have read their shared-memory source.
__device__ __forceinline__ void bulk_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
// Wait until this thread's bulk stores are complete.
__device__ __forceinline__ void bulk_wait_all() {
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}
// GPU-scope acquire-release fence: this thread's earlier global writes are
// visible to any thread that later synchronises with it at GPU scope (the
// split-KV arrival count), and the other way round for later reads.
__device__ __forceinline__ void fence_gpu() { asm volatile("fence.acq_rel.gpu;" ::: "memory"); }
// Make this thread's shared-memory writes visible to the async (TMA) proxy.
__device__ __forceinline__ void fence_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ----------------------------------------------------------------- tcgen05
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Warp-wide forms: every lane of the MMA warp runs the issue loop (so the
// operands are warp-uniform) and elect.sync picks the one lane that issues.
__device__ __forceinline__ void tc_commit_e(uint32_t bar) {
    asm volatile(
        "{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
        "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(bar)
        : "memory");
}
__device__ __forceinline__ void mma_ss_e(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc,
                                         uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred e, p;\n\telect.sync _|e, 0xffffffff;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
        "l"(a), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}
__device__ __forceinline__ void mma_ts_e(uint32_t d, uint32_t a, uint64_t b, uint32_t idesc,
                                         uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred e, p;\n\telect.sync _|e, 0xffffffff;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d),
        "r"(a), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}

#define PV_R8(i) "=r"(r[i]), "=r"(r[i + 1]), "=r"(r[i + 2]), "=r"(r[i + 3]), "=r"(r[i + 4]), \
                 "=r"(r[i + 5]), "=r"(r[i + 6]), "=r"(r[i + 7])
#define PV_W8(i) "r"(r[i]), "r"(r[i + 1]), "r"(r[i + 2]), "r"(r[i + 3]), "r"(r[i + 4]), \
                 "r"(r[i + 5]), "r"(r[i + 6]), "r"(r[i + 7])

// 32 / 128 consecutive TMEM columns of this thread's lane.  The wait for
// the load sits in the same asm statement, so no use of the registers can be
// scheduled before the data has arrived.
__device__ __forceinline__ void tmem_ld32_wait(uint32_t taddr, uint32_t* r) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
}
__device__ __forceinline__ void tmem_ld128_wait(uint32_t taddr, uint32_t* r) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x128.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63,%64,%65,%66,%67,%68,%69,%70,%71,%72,%73,%74,%75,%76,%77,%78,%79,%80,%81,%82,%83,%84,%85,%86,%87,%88,%89,%90,%91,%92,%93,%94,%95,%96,%97,%98,%99,%100,%101,%102,%103,%104,%105,%106,%107,%108,%109,%110,%111,%112,%113,%114,%115,%116,%117,%118,%119,%120,%121,%122,%123,%124,%125,%126,%127}, [%128];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]), "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63]), "=r"(r[64]), "=r"(r[65]), "=r"(r[66]), "=r"(r[67]), "=r"(r[68]), "=r"(r[69]), "=r"(r[70]), "=r"(r[71]), "=r"(r[72]), "=r"(r[73]), "=r"(r[74]), "=r"(r[75]), "=r"(r[76]), "=r"(r[77]), "=r"(r[78]), "=r"(r[79]), "=r"(r[80]), "=r"(r[81]), "=r"(r[82]), "=r"(r[83]), "=r"(r[84]), "=r"(r[85]), "=r"(r[86]), "=r"(r[87]), "=r"(r[88]), "=r"(r[89]), "=r"(r[90]), "=r"(r[91]), "=r"(r[92]), "=r"(r[93]), "=r"(r[94]), "=r"(r[95]), "=r"(r[96]), "=r"(r[97]), "=r"(r[98]), "=r"(r[99]), "=r"(r[100]), "=r"(r[101]), "=r"(r[102]), "=r"(r[103]), "=r"(r[104]), "=r"(r[105]), "=r"(r[106]), "=r"(r[107]), "=r"(r[108]), "=r"(r[109]), "=r"(r[110]), "=r"(r[111]), "=r"(r[112]), "=r"(r[113]), "=r"(r[114]), "=r"(r[115]), "=r"(r[116]), "=r"(r[117]), "=r"(r[118]), "=r"(r[119]), "=r"(r[120]), "=r"(r[121]), "=r"(r[122]), "=r"(r[123]), "=r"(r[124]), "=r"(r[125]), "=r"(r[126]), "=r"(r[127])
        : "r"(taddr)
        : "memory");
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t* r) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        PV_W8(0), PV_W8(8), PV_W8(16), PV_W8(24)
        : "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor: start, leading / stride byte offsets,
// version 1 (sm_100), 128-byte swizzle.
__device__ __forceinline__ uint64_t sdesc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((addr >> 4) & 0x3FFF) | ((uint64_t)((lbo >> 4) & 0x3FFF) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFF) << 32) | (1ull << 46) | (2ull << 61);
}

// Instruction descriptor of kind::f16: bf16 A and B, f32 accumulator, A
// K-major, B K-major or MN-major, M x N.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool b_mn_major) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((b_mn_major ? 1u : 0u) << 16) |
           ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&b);
}


// ----------------------------------------------------------------- schedule
// Stream-K: CTA c owns the key tiles [bound(c), bound(c+1)) of the launch's
// item list (see pv_plan.cu).  A segment is the part of one item inside that
// range.  Whole items at run time: every segment is a whole item.
__device__ __forceinline__ long long bound(const AttnParams& p, int c) {
    return (long long)c * p.total / p.grid;
}
// The CTA whose range holds key tile x.
__device__ __forceinline__ int cta_of(const AttnParams& p, long long x) {
    return (int)(((x + 1) * p.grid - 1) / p.total);
}

struct Seg {
    int si, head, qb, kt0, n, q0, rows[2];
    int item;      // global item index
    long long i0;  // the item's first key tile in the launch's tile sequence
    int c_first;   // first CTA holding part of the item
    int nseg;      // CTAs holding parts of the item
    int which;     // 0: this CTA's first segment, 1: a later one
};

// The whole item `item` as one segment (items handed out at run time).
__device__ __forceinline__ void item_seg(const AttnParams& p, int item, Seg& g) {
    int i = 0;
    while (i + 1 < p.n_streams && p.st[i + 1].item0 <= item) ++i;
    const AttnStreamDesc& s = p.st[i];
    const int li = item - s.item0;
    g.si = i;
    g.kt0 = 0;
    g.n = s.n_kt;
    g.qb = li / p.heads;
    g.head = li - g.qb * p.heads;
    g.item = item;
    g.i0 = s.cost0 + (long long)li * s.n_kt;
    g.c_first = blockIdx.x;
    g.nseg = 1;
    g.which = 0;
    g.q0 = g.qb * kQBlock;
    g.rows[0] = min(kQRows, s.n_q - g.q0);
    g.rows[1] = max(0, min(kQRows, s.n_q - g.q0 - kQRows));
}

struct SegIter {
    long long pos, end;
    __device__ SegIter(const AttnParams& p) : pos(bound(p, blockIdx.x)), end(bound(p, blockIdx.x + 1)) {}
    __device__ bool next(const AttnParams& p, Seg& g) {
        if (pos >= end) return false;
        int i = 0;
        while (i + 1 < p.n_streams && p.st[i + 1].cost0 <= pos) ++i;
        const AttnStreamDesc& s = p.st[i];
        const long long off = pos - s.cost0;
        const int li = (int)(off / s.n_kt);
        g.si = i;
        g.kt0 = (int)(off - (long long)li * s.n_kt);
        const long long i0 = s.cost0 + (long long)li * s.n_kt;   // the item's key-tile range
        const long long i1 = i0 + s.n_kt;
        const long long e = i1 < end ? i1 : end;
        g.n = (int)(e - pos);
        g.which = pos == bound(p, blockIdx.x) ? 0 : 1;
        // items are laid out query-block-major: with a grid that is a multiple
        // of n_qb, the CTAs working on one head's query blocks then walk the
        // same key tiles at the same time and share them through L2
        g.qb = li / p.heads;
        g.head = li - g.qb * p.heads;
        g.item = s.item0 + li;
        g.i0 = i0;
        g.c_first = cta_of(p, i0);
        g.nseg = cta_of(p, i1 - 1) - g.c_first + 1;
        g.q0 = g.qb * kQBlock;
        g.rows[0] = min(kQRows, s.n_q - g.q0);
        g.rows[1] = max(0, min(kQRows, s.n_q - g.q0 - kQRows));
        pos = e;
        return true;
    }
};

// Items handed out at run time.  The producer thread takes the next item
// index from counters[0] and passes it to the MMA warp and the eight softmax
// warps through a ring of kRing shared-memory slots; -1 ends the list.
// Slot k is written once the consumers have all released slot k - kRing.
__device__ bool item_grab(const AttnParams& p, Bars* b, int& k, Seg& g, bool& ok) {
    const int s = k % kRing;
    if (k >= kRing && !(ok = mbar_wait(smem_u32(&b->ring_empty[s]), ((k / kRing) - 1) & 1, b, p.err)))
        return false;
    int item = atomicAdd(p.counters, 1);
    if (item >= p.n_items) item = -1;
    *(volatile int*)&b->ring[s] = item;
    mbar_arrive(smem_u32(&b->ring_full[s]));  // release: the slot's value is visible
    ++k;
    if (item < 0) return false;
    item_seg(p, item, g);
    return true;
}
// Warp-wide: the next slot of the ring.
__device__ bool item_take(const AttnParams& p, Bars* b, int& k, Seg& g, bool& ok) {
    const int s = k % kRing;
    ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&b->ring_full[s]), (k / kRing) & 1, b, p.err));
    if (!ok) return false;
    const int item = *(volatile int*)&b->ring[s];
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(smem_u32(&b->ring_empty[s]));
    ++k;
    if (item < 0) return false;
    item_seg(p, item, g);
    return true;
}

// Partial slot of CTA c's part of an item starting at key tile i0, tile X.
__device__ __forceinline__ size_t part_slot(const AttnParams& p, int c, long long i0, int X) {
    const int which = i0 <= bound(p, c) ? 0 : 1;
    return ((size_t)c * 2 + which) * 2 + X;
}

// ----------------------------------------------------------------- roles
template <int D, bool kRun>
__device__ void producer(const CUtensorMap* tq, const CUtensorMap* tk, const CUtensorMap* tv,
                         const AttnParams& p, uint8_t* smem, Bars* b) {
    using C = Cfg<D>;
    const uint32_t qbar = smem_u32(&b->q_full);
    int kv = 0, qseg = 0;
    int ev0 = 0;              // first release event of the current segment
    int stage_ev[C::kStages]; // release event of the tile in each stage
    bool ok = true;
    int rk = 0;  // ring slots written
    SegIter it(p);
    Seg g;
    while (ok && (kRun ? item_grab(p, b, rk, g, ok) : it.next(p, g))) {
        const AttnStreamDesc& s = p.st[g.si];
        const int ntile = g.rows[1] > 0 ? 2 : 1;
        // the previous segment's S products are done with the Q tiles
        if (!(ok = mbar_wait(smem_u32(&b->q_empty), (qseg & 1) ^ 1, b, p.err))) break;
        mbar_expect_tx(qbar, ntile * C::kTileBytes);
        const int qrow = s.q_row0 + g.head * s.n_q + g.q0;
        for (int t = 0; t < ntile; ++t)
            for (int c = 0; c < C::kSub; ++c)
                tma_load(smem_u32(smem + C::kQOff + t * C::kTileBytes + c * 16384), tq, c * 64,
                         qrow + t * kQRows, qbar);
        ++qseg;
        const int krow0 = s.kv_row0 + g.head * s.kv_head_stride + g.kt0 * kKeyTile;
        for (int j = 0; ok && j < g.n; ++j) {
            for (int w = 0; w < 2; ++w) {
                const int st = kv % C::kStages;
                // the tile loaded kStages loads ago must have been released
                if (kv >= C::kStages) {
                    const int e = stage_ev[st];
                    if (!(ok = mbar_wait(smem_u32(&b->rel[e & 7]), (e >> 3) & 1, b, p.err))) break;
                }
                // K_j is released at the end of iteration j, V_j at the end of
                // iteration j + 1 (or of the segment)
                stage_ev[st] = ev0 + j + w;
                const uint32_t full = smem_u32(&b->kv_full[st]);
                mbar_expect_tx(full, C::kTileBytes);
                const CUtensorMap* m = w == 0 ? tk : tv;
                for (int c = 0; c < C::kSub; ++c)
                    tma_load(smem_u32(smem + C::kKVOff + st * C::kTileBytes + c * 16384), m,
                             c * 64, krow0 + j * kKeyTile, full);
                ++kv;
            }
        }
        ev0 += g.n + 1;
    }
    // Before leaving, make sure no copy of ours is still landing in shared
    // memory: wait (bounded) for the last load issued into each stage, and
    // for the last Q load.
    for (int idx = max(0, kv - C::kStages); idx < kv; ++idx) {
        const uint32_t bar = smem_u32(&b->kv_full[idx % C::kStages]);
        const uint32_t ph = (idx / C::kStages) & 1;
        const long long t0 = clock64();
        while (!mbar_try(bar, ph) && clock64() - t0 < kWaitCycles) {
        }
    }
    if (qseg > 0) {
        const long long t0 = clock64();
        while (!mbar_try(qbar, (qseg - 1) & 1) && clock64() - t0 < kWaitCycles) {
        }
    }
}

template <int D, bool kRun>
__device__ void mma_issuer(const AttnParams& p, uint8_t* smem, Bars* b, uint32_t tmem) {
    using C = Cfg<D>;
    // every lane waits; the vote reconverges the warp before the next issue
    auto wwait = [&](uint32_t bar, uint32_t par, Bars* bb, int* err) -> bool {
        const bool r = mbar_wait(bar, par, bb, err);
        return __all_sync(0xffffffffu, r);
    };
    constexpr uint32_t idesc_qk = idesc_bf16(kQRows, kKeyTile, false);
    constexpr uint32_t idesc_pv = idesc_bf16(kQRows, D, true);
    const uint32_t sQ = smem_u32(smem + C::kQOff);
    const uint32_t sKV = smem_u32(smem + C::kKVOff);
    auto qk = [&](int X, int stage) {
        const uint32_t tS = tmem + X * 128;
        const uint32_t qa = sQ + X * C::kTileBytes;
        const uint32_t kb = sKV + stage * C::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
            mma_ss_e(tS, sdesc(qa + off, 16, 1024), sdesc(kb + off, 16, 1024), idesc_qk, kk > 0);
        }
    };
    auto pv = [&](int X, int stage, bool acc, int k0) {
        const uint32_t tS = tmem + X * 128;
        const uint32_t tO = tmem + C::kColsO + X * D;
        const uint32_t vb = sKV + stage * C::kTileBytes;
#pragma unroll
        for (int kk = k0; kk < k0 + kKeyTile / 32; ++kk)
            mma_ts_e(tO, tS + kk * 8, sdesc(vb + kk * 2048, 16384, 1024), idesc_pv,
                   (acc || kk > 0) ? 1u : 0u);
    };
    int kv = 0, qseg = 0;
    int ev0 = 0;         // first release event of the current segment
    int pc[2] = {0, 0};  // P tiles consumed, per query tile
    int oc[2] = {0, 0};  // segments finished, per query tile
    bool ok = true;
    // P V of tile X for key tile j of the current segment; the first one of
    // a segment overwrites O, which the previous segment's epilogue must
    // have read out first.
    auto do_pv = [&](int X, int stage, int j) -> bool {
        if (j == 0 && !wwait(smem_u32(&b->o_empty[X]), (oc[X] & 1) ^ 1, b, p.err)) return false;
        if (!wwait(smem_u32(&b->p_lo[X]), pc[X] & 1, b, p.err)) return false;
        tc_fence_after();
        pv(X, stage, j > 0, 0);          // keys 0..63 while the softmax does 64..127
        if (!wwait(smem_u32(&b->p_full[X]), pc[X] & 1, b, p.err)) return false;
        ++pc[X];
        tc_fence_after();
        pv(X, stage, true, kKeyTile / 32);
        return true;
    };
    int rk = 0;  // ring slots taken
    SegIter it(p);
    Seg g;
    while (ok && (kRun ? item_take(p, b, rk, g, ok) : it.next(p, g))) {
        const bool hasB = g.rows[1] > 0;
        if (!(ok = wwait(smem_u32(&b->q_full), qseg & 1, b, p.err))) break;
        ++qseg;
        tc_fence_after();
        const int n = g.n;
        for (int j = 0; ok && j < n; ++j) {
            const int ks = (kv + 2 * j) % C::kStages;
            const uint32_t kph = ((kv + 2 * j) / C::kStages) & 1;
            const int vs_prev = (kv + 2 * j - 1) % C::kStages;
            const uint32_t vph_prev = ((kv + 2 * j - 1) / C::kStages) & 1;
            if (j > 0) {
                if (!(ok = wwait(smem_u32(&b->kv_full[vs_prev]), vph_prev, b, p.err) &&
                           do_pv(0, vs_prev, j - 1)))
                    break;
            }
            if (!(ok = wwait(smem_u32(&b->kv_full[ks]), kph, b, p.err))) break;
            tc_fence_after();
            qk(0, ks);
            tc_commit_e(smem_u32(&b->s_full[0]));
            if (hasB) {
                if (j > 0 && !(ok = do_pv(1, vs_prev, j - 1))) break;
                qk(1, ks);
                tc_commit_e(smem_u32(&b->s_full[1]));
            }
            // one release per iteration: K_j and V_(j-1) are no longer read
            tc_commit_e(smem_u32(&b->rel[(ev0 + j) & 7]));
        }
        if (!ok) break;
        tc_commit_e(smem_u32(&b->q_empty));  // the Q tiles are free once these S products end
        const int vs = (kv + 2 * n - 1) % C::kStages;
        const uint32_t vph = ((kv + 2 * n - 1) / C::kStages) & 1;
        if (!(ok = wwait(smem_u32(&b->kv_full[vs]), vph, b, p.err) && do_pv(0, vs, n - 1)))
            break;
        tc_commit_e(smem_u32(&b->o_full[0]));
        ++oc[0];
        if (hasB) {
            if (!(ok = do_pv(1, vs, n - 1))) break;
            tc_commit_e(smem_u32(&b->o_full[1]));
            ++oc[1];
        }
        tc_commit_e(smem_u32(&b->rel[(ev0 + n) & 7]));  // V of the last iteration
        kv += 2 * n;
        ev0 += n + 1;
    }
    // every MMA issued by this thread has completed once mma_done flips
    tc_commit_e(smem_u32(&b->mma_done));
    const long long t0 = clock64();
    while (!mbar_try(smem_u32(&b->mma_done), 0) && clock64() - t0 < kWaitCycles) {
    }
    __syncwarp();
}

// Exponentials of 64 of this thread's scores: p = 2^(s*sl2 - m) on the XU
// pipe, written to TMEM as bf16 pairs at tP (32 columns, one store; fewer,
// larger stores than 16-column ones measured 4 % faster per launch).  The
// bf16 value is the upper half of the f32 (round toward zero, a byte permute
// on the ALU pipe instead of a conversion on the XU pipe); the returned sum
// adds exactly those rounded values, so that P and its normaliser agree.
__device__ __forceinline__ float exp_half(const uint32_t* sr, float2 sl2x2, float2 nmx2,
                                          uint32_t tP) {
    float2 acc[4] = {{0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}};
    uint32_t pk[32];
#pragma unroll
    for (int i = 0; i < 64; i += 2) {
        const float2 x = __ffma2_rn(make_float2(__uint_as_float(sr[i]), __uint_as_float(sr[i + 1])),
                                    sl2x2, nmx2);
        const uint32_t b0 = __float_as_uint(ex2(x.x)) & 0xFFFF0000u;
        const uint32_t b1 = __float_as_uint(ex2(x.y)) & 0xFFFF0000u;
        acc[(i >> 1) & 3] =
            __fadd2_rn(acc[(i >> 1) & 3], make_float2(__uint_as_float(b0), __uint_as_float(b1)));
        pk[i / 2] = __byte_perm(b0, b1, 0x7632);
    }
    tmem_st32(tP, pk);
    const float2 a = __fadd2_rn(__fadd2_rn(acc[0], acc[1]), __fadd2_rn(acc[2], acc[3]));
    return a.x + a.y;
}

// Row maximum of 128 scores (masked ones are -inf).
__device__ __forceinline__ float row_max(const uint32_t* sr) {
    float mx8[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) mx8[i] = __uint_as_float(sr[i]);
#pragma unroll
    for (int c = 8; c < 128; c += 16)
#pragma unroll
        for (int i = 0; i < 8; ++i)
            mx8[i] = fmax3(mx8[i], __uint_as_float(sr[c + i]), __uint_as_float(sr[c + 8 + i]));
    return fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]),
                 fmaxf(mx8[6], mx8[7]));
}

// Normalised bf16 output of 32 f32 columns: row dst[0..32) = o * inv.
__device__ __forceinline__ void store_row32(bf16* dst, const uint32_t* o, float inv) {
    uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int q = i * 8;
        d4[i] = make_uint4(
            pack_bf16(__uint_as_float(o[q + 0]) * inv, __uint_as_float(o[q + 1]) * inv),
            pack_bf16(__uint_as_float(o[q + 2]) * inv, __uint_as_float(o[q + 3]) * inv),
            pack_bf16(__uint_as_float(o[q + 4]) * inv, __uint_as_float(o[q + 5]) * inv),
            pack_bf16(__uint_as_float(o[q + 6]) * inv, __uint_as_float(o[q + 7]) * inv));
    }
}

// Coalesced output.  One thread holds one query row, and rows of one head are
// 6 KB apart in out[token][head][D], so direct stores touch 32 cache lines per
// warp instruction.  Instead a warp whose 32 rows are all queries puts its
// rows into its own shared-memory buffer (32 rows x 64 columns of bf16, the
// 16-byte chunk k of row r at chunk k ^ (r & 7): the 128-byte swizzle of the
// output tensor map, and free of bank conflicts) and one TMA store writes the
// block as whole 128-byte row pieces.
// Columns 32h .. 32h+31 of the staged 64-column block, scaled by `scale`.
__device__ __forceinline__ void stage_put32(uint8_t* buf, int h, const uint32_t* o, float scale) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int q = i * 8;
        const int k = h * 4 + i;
        *reinterpret_cast<uint4*>(buf + lane * 128 + ((k ^ (lane & 7)) << 4)) = make_uint4(
            pack_bf16(__uint_as_float(o[q + 0]) * scale, __uint_as_float(o[q + 1]) * scale),
            pack_bf16(__uint_as_float(o[q + 2]) * scale, __uint_as_float(o[q + 3]) * scale),
            pack_bf16(__uint_as_float(o[q + 4]) * scale, __uint_as_float(o[q + 5]) * scale),
            pack_bf16(__uint_as_float(o[q + 6]) * scale, __uint_as_float(o[q + 7]) * scale));
    }
}
// Before the buffer is written again: the warp's previous store has read it.
__device__ __forceinline__ void stage_acquire() {
    if ((threadIdx.x & 31) == 0) bulk_wait_read();
    __syncwarp();
}
// The staged block to out: columns c0 .. c0+63 of `head` for tokens tok0 ..
// tok0+31, one TMA store issued by lane 0.
__device__ __forceinline__ void stage_flush(const CUtensorMap* to, const uint8_t* buf, int c0,
                                            int head, int tok0) {
    fence_async_smem();
    __syncwarp();
    if ((threadIdx.x & 31) == 0) tma_store_3d(to, smem_u32(buf), c0, head, tok0);
}

// Merge of the split parts of one query tile by the last CTA to arrive
// (split-KV combination of the online softmax: with M = max_k m_k and
// L = sum_k l_k 2^(m_k - M), o = sum_k O_k 2^(m_k - M) / L).  Part k sits in
// the partial slot of CTA c_first + k; with `keep` this CTA's own part is
// still in TMEM (tO, m_own, l_own) and is taken from there, bit for bit the
// values it stored.  Sums run in part order whichever CTA merges, so results
// are reproducible.  The (m, l) loads are issued four parts at a time (one
// pass) and a part's 32-column block in one batch: a merge costs a few L2
// round trips.
// Split-KV partial rows go to L2 with an evict-last policy, so that the
// key / value stream of the launch does not push them to DRAM before the
// last CTA to arrive merges them; that CTA then drops each merged line
// without writing it back (the next launch writes a slot before it reads
// it).  Without this about half of the parts written early in a CTA's run
// went to DRAM and came back; with it the launch's DRAM writes are its
// output.
__device__ __forceinline__ unsigned long long l2_keep_policy() {
    unsigned long long pol;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}
__device__ __forceinline__ void st_keep(float* a, float v, unsigned long long pol) {
    asm volatile("st.global.cg.L2::cache_hint.f32 [%0], %1, %2;" ::"l"(a), "f"(v), "l"(pol)
                 : "memory");
}
// Drops the 128-byte L2 line at a (128-byte aligned) without writing it
// back; `after` is computed from the line's data, so that the drop is
// issued after the line was read.
__device__ __forceinline__ void l2_discard(const float* a, float after) {
    asm volatile("discard.global.L2 [%0], 128;" ::"l"(a), "f"(after) : "memory");
}

template <int D>
__device__ __forceinline__ void merge_parts(const AttnParams& p, const Seg& g, int X, int r,
                                            bool row_ok, bool keep, uint32_t tO, float m_own,
                                            float l_own, bf16* dst, float* lse_dst,
                                            const CUtensorMap* to, uint8_t* ebuf, bool warp_full,
                                            int tok_w) {
    const size_t slot_f = partial_slot_floats(D);
    const int self = keep ? (int)blockIdx.x - g.c_first : -1;
    auto ml = [&](int k) -> const float* {
        return p.partial + part_slot(p, g.c_first + k, g.i0, X) * slot_f + (size_t)kQRows * D;
    };
    // running (M, L) over the parts in order, L relative to M: one batch of
    // loads per four parts
    float M = -INFINITY, L = 0.f;
    for (int k0 = 0; k0 < g.nseg; k0 += 4) {
        float mk[4], lk[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int k = k0 + u;
            mk[u] = k == self ? m_own : (k < g.nseg ? __ldcg(ml(k) + r) : -INFINITY);
            lk[u] = k == self ? l_own : (k < g.nseg ? __ldcg(ml(k) + kQRows + r) : 0.f);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            if (k0 + u < g.nseg) {
                const float Mn = fmaxf(M, mk[u]);
                L = L * ex2(M - Mn) + lk[u] * ex2(mk[u] - Mn);
                M = Mn;
            }
        }
    }
    const float invL = 1.0f / L;
#pragma unroll 1
    for (int c = 0; c < D; c += 32) {
        float acc[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) acc[i] = 0.f;
        for (int k = 0; k < g.nseg; ++k) {
            uint32_t v[32];
            float w;
            if (k == self) {
                tmem_ld32_wait(tO + c, v);
                w = ex2(m_own - M) * invL;
            } else {
                const float* pk = ml(k) - (size_t)kQRows * D;
                w = ex2(__ldcg(pk + (size_t)kQRows * D + r) - M) * invL;
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    v[i] = __float_as_uint(__ldcg(pk + (size_t)(c + i) * kQRows + r));
            }
#pragma unroll
            for (int i = 0; i < 32; ++i) acc[i] = fmaf(w, __uint_as_float(v[i]), acc[i]);
        }
        uint32_t o[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(acc[i]);
        if (warp_full) {
            if ((c & 63) == 0) stage_acquire();
            stage_put32(ebuf, (c >> 5) & 1, o, 1.0f);
            if ((c & 63) == 32) stage_flush(to, ebuf, c - 32, g.head, tok_w);
        } else if (row_ok) {
            store_row32(dst + c, o, 1.0f);
        }
    }
    if (row_ok && lse_dst) *lse_dst = (M + __log2f(L)) * 0.69314718055994531f;
    // every part's lines of this warp's 32 rows (the merging CTA's own part
    // too: it was written before the arrival count and read from TMEM): a
    // line per lane and 32 columns, then the m and l lines
    for (int k = 0; k < g.nseg; ++k) {
        const float* pk = ml(k) - (size_t)kQRows * D;
        for (int c = 0; c < D; c += 32)
            l2_discard(pk + (size_t)(c + (r & 31)) * kQRows + (r & ~31), L);
        if ((r & 31) < 2) l2_discard(ml(k) + (r & 31) * kQRows + (r & ~31), L);
    }
}

template <int D, bool kRun>
__device__ void softmax_epilogue(const AttnParams& p, const CUtensorMap* to, uint8_t* smem,
                                 Bars* b, uint32_t tmem, int X) {
    using C = Cfg<D>;
    const int wq = (threadIdx.x / 32) & 3;          // TMEM lane quadrant of this warp
    const int r = wq * 32 + (threadIdx.x & 31);     // query row inside the tile
    const uint32_t lane = (uint32_t)(wq * 32) << 16;
    const uint32_t tS = tmem + lane + X * 128;
    const uint32_t tO = tmem + lane + C::kColsO + X * D;
    uint8_t* ebuf = smem + C::kEpiOff + (X * 4 + wq) * C::kEpiWarpBytes;  // this warp's staging
    const float sl2 = p.scale_log2;
    const float ln2 = 0.69314718055994531f;
    const size_t slot_f = partial_slot_floats(D);
    int sc = 0;   // S tiles taken, for the s_full phase
    int oc = 0;   // segments finished, for the o_full phase
    int ec = 0;   // split epilogues, for the ep_in / ep_out phases
    bool ok = true;
    int rk = 0;  // ring slots taken
    SegIter it(p);
    Seg g;
    while (ok && (kRun ? item_take(p, b, rk, g, ok) : it.next(p, g))) {
        if (g.rows[X] == 0) continue;  // this segment has no query tile X
        const AttnStreamDesc& s = p.st[g.si];
        float m = -INFINITY;  // maximum applied to the exponentials, log2 units
        float l = 0.f;        // sum of the exponentials (as rounded into P)
        for (int j = 0; j < g.n; ++j) {
            ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&b->s_full[X]), sc & 1, b, p.err));
            if (!ok) break;
            ++sc;
            tc_fence_after();
            uint32_t sr[128];
            tmem_ld128_wait(tS, sr);
            const int valid = s.n_k - (g.kt0 + j) * kKeyTile;
            if (valid < kKeyTile) {
#pragma unroll
                for (int c = 0; c < 128; ++c)
                    if (c >= valid) sr[c] = __float_as_uint(-INFINITY);
            }
            {
                // the tile's row maximum; O is rescaled only when it grows by
                // more than 8 (log2 units), so p stays <= 2^8
                const float m_t = row_max(sr) * sl2;
                if (j == 0) {
                    m = m_t;
                } else if (__any_sync(0xffffffffu, m_t > m + 8.0f)) {
                    const float m_new = fmaxf(m, m_t);
                    const float alpha = ex2(m - m_new);
                    l *= alpha;
                    m = m_new;
                    // O holds P V of tiles < j, complete: S(j) was committed after it
#pragma unroll 1
                    for (int c = 0; c < D; c += 32) {
                        uint32_t o[32];
                        tmem_ld32_wait(tO + c, o);
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
                        tmem_st32(tO + c, o);
                    }
                }
            }
            // P in two halves: the first goes to the tensor pipe (P V of keys
            // 0..63) while the second half's exponentials are computed
            const float2 sl2x2 = make_float2(sl2, sl2);
            const float2 nmx2 = make_float2(-m, -m);
            l += exp_half(sr, sl2x2, nmx2, tS);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if ((threadIdx.x & 31) == 0) mbar_arrive(smem_u32(&b->p_lo[X]));
            l += exp_half(sr + 64, sl2x2, nmx2, tS + 32);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if ((threadIdx.x & 31) == 0) mbar_arrive(smem_u32(&b->p_full[X]));
        }
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&b->o_full[X]), oc & 1, b, p.err));
        ++oc;
        if (!ok) break;
        tc_fence_after();

        // ------------------------------------------------------ epilogue
        const bool row_ok = r < g.rows[X];
        const int tok = s.out_tok0 + g.q0 + X * kQRows + r;
        const bool whole = g.nseg == 1;
        // On the CTA's last segment O may stay in TMEM until the arrival
        // count says whether this CTA merges: the merge then reads its own
        // part from there instead of back from global memory.
        const bool keep = !whole && it.pos >= it.end;
        const float inv = 1.0f / l;
        bf16* dst = p.out + ((size_t)tok * p.heads + g.head) * D;
        float* mine = p.partial + part_slot(p, blockIdx.x, g.i0, X) * slot_f;
        const bool warp_full = wq * 32 + 31 < g.rows[X];  // all 32 rows of this warp are queries
        const int tok_w = s.out_tok0 + g.q0 + X * kQRows + wq * 32;
        // O leaves TMEM in 32-column chunks: to the output when this CTA
        // holds the whole item, else to this CTA's partial slot
        // (column-major [D][128], then m[128], l[128]: a warp stores 32
        // consecutive floats).
#pragma unroll 1
        for (int c = 0; c < D; c += 32) {
            uint32_t o[32];
            tmem_ld32_wait(tO + c, o);
            if (whole) {
                if (warp_full) {
                    if ((c & 63) == 0) stage_acquire();
                    stage_put32(ebuf, (c >> 5) & 1, o, inv);
                    if ((c & 63) == 32) stage_flush(to, ebuf, c - 32, g.head, tok_w);
                } else if (row_ok) {
                    store_row32(dst + c, o, inv);
                }
            } else {
                const unsigned long long pol = l2_keep_policy();
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    st_keep(mine + (size_t)(c + i) * kQRows + r, __uint_as_float(o[i]), pol);
            }
        }
        if (!keep) {
            // O is read out: the next segment's first P V may overwrite it
            tc_fence_before();
            __syncwarp();
            if ((threadIdx.x & 31) == 0) mbar_arrive(smem_u32(&b->o_empty[X]));
        }
        if (whole) {
            if (row_ok && p.lse) p.lse[(size_t)tok * p.heads + g.head] = (m + __log2f(l)) * ln2;
            continue;
        }
        {
            const unsigned long long pol = l2_keep_policy();
            st_keep(mine + (size_t)kQRows * D + r, m, pol);
            st_keep(mine + (size_t)kQRows * D + kQRows + r, l, pol);
        }
        // all four warps' partial rows are visible before the arrival count
        // moves; bounded waits on mbarriers, not bar.sync, so that an
        // aborting CTA can never block here
        fence_gpu();
        __syncwarp();
        if ((threadIdx.x & 31) == 0) mbar_arrive(smem_u32(&b->ep_in[X]));
        if (r == 0) {
            int last = 0;
            if (mbar_wait(smem_u32(&b->ep_in[X]), ec & 1, b, p.err) &&
                !*(volatile int*)&b->abort) {
                int* cnt = p.counters + (size_t)g.item * kQTilesPerCta + X;
                const int old = atomicAdd(cnt, 1);
                last = old == g.nseg - 1;
                if (last) *cnt = 0;  // ready for the next launch
            }
            b->last[X] = last;
            mbar_arrive(smem_u32(&b->ep_out[X]));
        }
        ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&b->ep_out[X]), ec & 1, b, p.err));
        ++ec;
        if (ok && b->last[X]) {
            fence_gpu();
            merge_parts<D>(p, g, X, r, row_ok, keep, tO, m, l, dst,
                           p.lse ? p.lse + (size_t)tok * p.heads + g.head : nullptr, to, ebuf,
                           warp_full, tok_w);
        }
        if (keep) {
            tc_fence_before();
            __syncwarp();
            if ((threadIdx.x & 31) == 0) mbar_arrive(smem_u32(&b->o_empty[X]));
        }
    }
    // this warp's output stores are complete before the CTA ends
    if ((threadIdx.x & 31) == 0) bulk_wait_all();
    __syncwarp();
}

// kRun: whole items handed out at run time (AttnParams::item_aligned == 1);
// otherwise stream-K.  Two instantiations, so that each keeps its own code.
template <int D, bool kRun>
__global__ void __launch_bounds__(kThreads, 1)
    attn_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap to,
                const __grid_constant__ AttnParams p) {
    using C = Cfg<D>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    Bars* b = reinterpret_cast<Bars*>(smem + C::kBarOff);
    const int warp = threadIdx.x / 32;
    const int lane_id = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&b->q_full), 1);
        mbar_init(smem_u32(&b->q_empty), 1);
        for (int x = 0; x < 2; ++x) {
            mbar_init(smem_u32(&b->s_full[x]), 1);
            mbar_init(smem_u32(&b->p_full[x]), 4);   // one arrive per softmax warp
            mbar_init(smem_u32(&b->p_lo[x]), 4);
            mbar_init(smem_u32(&b->o_full[x]), 1);
            mbar_init(smem_u32(&b->o_empty[x]), 4);  // one arrive per softmax warp
            mbar_init(smem_u32(&b->ep_in[x]), 4);
            mbar_init(smem_u32(&b->ep_out[x]), 1);
        }
        mbar_init(smem_u32(&b->mma_done), 1);
        for (int i = 0; i < C::kStages; ++i) mbar_init(smem_u32(&b->kv_full[i]), 1);
        for (int i = 0; i < 8; ++i) mbar_init(smem_u32(&b->rel[i]), 1);
        for (int i = 0; i < kRing; ++i) {
            mbar_init(smem_u32(&b->ring_full[i]), 1);
            mbar_init(smem_u32(&b->ring_empty[i]), 9);  // the MMA warp and 8 softmax warps
        }
        b->abort = 0;
        b->last[0] = b->last[1] = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(&b->tmem_base)),
                     "r"(512u)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = b->tmem_base;
    if (warp < 4) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsLow));
        if (warp == 0) {
            if (lane_id == 0) producer<D, kRun>(&tq, &tk, &tv, p, smem, b);
        } else if (warp == 1) {
            mma_issuer<D, kRun>(p, smem, b, tmem);  // the whole warp; one elected lane issues
        }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsHigh));
        softmax_epilogue<D, kRun>(p, &to, smem, b, tmem, warp / 4 - 1);
    }
    tc_fence_before();
    __syncthreads();
    if (kRun && threadIdx.x == 0) {
        // every CTA has stopped taking items once it gets here: the last one
        // to arrive returns the hand-out counter to zero for the next launch
        __threadfence();
        if (atomicAdd(p.counters + 1, 1) == p.grid - 1) {
            p.counters[0] = 0;
            p.counters[1] = 0;
        }
    }
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512u)
                     : "memory");
    }
}

template <int D, bool kRun>
cudaError_t launch_d(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                     const CUtensorMap& to, const AttnParams& p, cudaStream_t s) {
    using C = Cfg<D>;
    static std::atomic<unsigned long long> configured{0};
    const cudaError_t e = smem_limit_once(attn_kernel<D, kRun>, C::kSmem, configured);
    if (e != cudaSuccess) return e;
    attn_kernel<D, kRun><<<p.grid, kThreads, C::kSmem, s>>>(tq, tk, tv, to, p);
    return cudaGetLastError();
}

// One bounded wait on an mbarrier that nothing arrives on: it gives up after
// kWaitCycles, records the timeout in *err and returns, exactly as a wait of
// attn_kernel does; used to check the failure path without a GPU fault.
__global__ void wait_timeout_kernel(int* err) {
    __shared__ Bars b;
    if (threadIdx.x == 0) {
        b.abort = 0;
        mbar_init(smem_u32(&b.q_full), 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        mbar_wait(smem_u32(&b.q_full), 0, &b, err);
    }
}

}  // namespace

cudaError_t launch_wait_timeout_probe(int* err, cudaStream_t s) {
    wait_timeout_kernel<<<1, 32, 0, s>>>(err);
    return cudaGetLastError();
}

static_assert(sizeof(AttnParams) + 4 * sizeof(CUtensorMap) <= 4096,
              "attention kernel parameters beyond 4 KB");

cudaError_t launch_attn(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                        const CUtensorMap& to, const AttnParams& p, cudaStream_t s) {
    if (p.grid <= 0 || p.total <= 0) return cudaErrorInvalidValue;
    const bool run = p.item_aligned != 0;
    if (p.head_dim == 128)
        return run ? launch_d<128, true>(tq, tk, tv, to, p, s) : launch_d<128, false>(tq, tk, tv, to, p, s);
    if (p.head_dim == 64)
        return run ? launch_d<64, true>(tq, tk, tv, to, p, s) : launch_d<64, false>(tq, tk, tv, to, p, s);
    return cudaErrorInvalidValue;
}

}  // namespace pv
