// moe_decode.cu -- MoE FFN decode / speculative-verify step on packed
// ROCmFPX-style experts: one persistent kernel per layer.
//
// What it computes (sources by page title and section):
//  - ainomam.com, "APU 实现 token 自由…", section "Lucebox 的优化三板斧":
//    256 routed experts + 1 shared, 6 active per token; in the q-column verify
//    pass each packed weight is decoded once for all columns.
//  - m.mzlw.cn, "Lucebox专攻DeepSeek V4…", section "MoE 专家并行": top-6 plus
//    1 shared expert per layer.
//  - taozi.news, "DeepSeek V4 Flash 在 128GB 锐龙 AI MAX+ 上跑到 32 tok/s",
//    section "ROCmFPX：把 284B 权重压进 128 GB": FP2 gate/up, FP3 down blocks.
//  For each column t: y[t] = sum_j w[t][j] Wd_e (silu(Wg_e x) * (Wu_e x)) + the
//  shared expert, e = idx[t][j].
//
// B200 design:
//  - Grouping: every CTA derives the union of routed experts over the T
//    columns (the "slots") from idx, so each expert is streamed once for all
//    the columns routed to it; slot 0 is the shared expert (all columns).
//  - One persistent kernel, one CTA per SM.  Gate/up units of 32 rows of I
//    (two 16-row row-groups) of every slot, slot-major, are dealt round-robin
//    (CTA b takes b, b + G, ...); then groups of 4 consecutive down row-groups
//    of every slot (one h image serves the group), slot-major, also
//    round-robin, offset so that the CTAs with an extra gate/up unit do not
//    also get an extra down group.  Every CTA thus
//    walks both phases slot by slot, and reaches a slot's down rows about when
//    the whole grid has finished that slot's gate/up rows.  The shared expert
//    does not depend on the routing: its first gate/up unit streams into
//    shared memory before the kernel waits for the router.
//  - No grid barrier between the gate/up and the down phase: a slot's down
//    rows need only that slot's h.  The epilogue of a gate/up unit writes the
//    down projection's B operand for its 32 values of I directly: per column a
//    power-of-two exponent n chosen from the unit's max |h|, the fp16 hi/lo
//    pair of h * 2^n in fragment order, the 16-row sums and 2^-n (folded into
//    the weight scale of the matching down tiles, so every h in the fp32 range
//    is carried to about 2^-22).  It then counts the unit done for its slot
//    (one fence and release reduction for the units stored since the last
//    count, issued when the epilogue warp would otherwise wait).  A CTA
//    streams a slot's down rows after one bulk copy of that image; both phases
//    run slot-major, so slots are ready long before their down rows come up.
//  - Per CTA: one lane of the producer warp streams spans of 8 chunks HBM ->
//    shared memory with 1-D bulk copies (TMA, evict-first L2 policy) into a
//    ring of stages, each with a record of what it holds (8 gate + 8 up
//    chunks, or two down row-groups).  8 consumer warps take one chunk of each
//    half of every stage, decode it in registers (one AND per A register, see
//    rfx_tile.cuh) and run mma.sync m16n8k16 in fp16: x normalised per column
//    by a power of two for gate/up, the scaled hi/lo split of h for down.  3
//    epilogue warps take the reduction units (a gate/up unit, or the one or
//    two down row-groups of a stage) in turn, sum the 8 warps' partials in a
//    fixed order and run SwiGLU and the h image (gate/up) or store the slot's
//    partial output (down).
//  - One grid barrier at the end, then the fixed-order weighted combine.
//  - Every wait is bounded; a timeout sets a workspace error flag, the CTA
//    drains its in-flight copies and exits.
#include <cuda_runtime.h>

#include "launch_util.h"
#include "moe_decode.h"
#include "rfx_tile.cuh"

namespace rfx {

constexpr int NCW = 8;                       // consumer warps 0..7
constexpr int WARP_PRODUCER = NCW;           // weight and h bulk copies (one lane)
constexpr int WARP_EPI0 = NCW + 1;           // epilogue warps: reductions, SwiGLU + h image / partial stores
constexpr int NEPI = 3;
constexpr int NWARPS = WARP_EPI0 + NEPI;
constexpr int NTHREADS = NWARPS * 32;
constexpr int NSTAGE_THREADS = NTHREADS - 32;  // every warp but the producer stages x
constexpr int NRED_MAX = MOE_MAX_RED;
constexpr long long DEFAULT_WAIT = 4000000000LL;
static_assert(MOE_MAX_RED % NEPI == 0, "reduction buffers are taken by the epilogue warps in turn");

struct __align__(16) SlotTable {
    float w[MOE_MAXT][MOE_MAXK];              // routing weights
    signed char tslot[MOE_MAXT][MOE_MAXK];    // slot of (column, j), -1 if invalid
    signed char tpos[MOE_MAXT][MOE_MAXK];     // position of the column among the slot's columns
    int nslots;
    int expert[MOE_MAXS];                     // -1: shared expert
    int ncols[MOE_MAXS];
    unsigned colmask[MOE_MAXS];               // columns routed to the slot (bit c)
    signed char cols[MOE_MAXS][MOE_MAXT];
    signed char fa[MOE_MAXS];                 // gate/up format of the slot
    signed char fb[MOE_MAXS];                 // down format
    signed char ci[MOE_MAXS];                 // staged x copy its gate/up tiles read
    unsigned mask[32];                        // experts in use (bit per expert)
    int prefix[32];
    int idx[MOE_MAXT * MOE_MAXK];
};

// A reduction unit: the 8 consumer warps' partials of one or two row-groups
// (a gate/up unit: always two; a down stage: its one or two), or the
// end-of-work marker.
enum : int { UNIT_A = 0, UNIT_B = 1, UNIT_END = 3 };
struct RedInfo {
    int kind, slot, ncols, rg, n;
};

// What a ring stage holds, written by the producer with the stage.
enum : short { REC_FIRST = 1, REC_LAST = 2, REC_HNEW = 4, REC_CLOSE = 8, REC_END = 16 };
struct __align__(16) StageRec {
    short kind;    // 0: gate + up span, 1: down span(s), -1: end of work
    short slot;
    short rg;      // row-group of the matrix (rows 16*rg ..); down: first of n
    short c0;      // first chunk of the span
    short n;       // down: row-groups in the stage (one per half); gate/up: half of the unit (rg & 1)
    short flags;   // REC_*: first / last span of the row-group(s); the deposit closes the reduction
                   // unit; a new slot's h in buffer hbuf
    short hbuf;    // down: shared-memory h buffer of the slot
    short pad;
};

struct Shared {
    uint64_t full[MOE_MAX_STAGES];
    uint64_t empty[MOE_MAX_STAGES];
    uint64_t hfull[2], hfree[2];
    uint64_t rfull[NRED_MAX], rempty[NRED_MAX];
    RedInfo rinfo[NRED_MAX];
    StageRec rec[MOE_MAX_STAGES];
    volatile int abort_flag;
    volatile int consumed;   // stages released by all consumer warps (for the abort drain)
    int bar_ok;
    unsigned xmax[MOE_MAXT]; // max |x| per column (fp32 bits)
    int xn[MOE_MAXT];        // x is staged as x * 2^xn[c] (then 2^-s_b per tile position)
    double rms_part[MOE_MAXT][8];   // chained input: per-warp sums of squares
    double rms_r[MOE_MAXT], rms_ri[MOE_MAXT];   // its RMS per column and 1 / RMS
    SlotTable st;
};

__device__ __forceinline__ void set_error(uint32_t* ctrl, uint32_t bits) { atomicOr(ctrl + MOE_CTRL_ERR, bits); }

// --------------------------------------------------------------- routing ---

// The routing of the T columns, loaded by the producer warp's lanes (lane L
// holds entries L and L + 32 of idx / w).
struct Routing {
    int e0, e1;
    float w0, w1;
};

__device__ __forceinline__ Routing load_routing(const MoeParams& p) {
    const int lane = threadIdx.x & 31;
    const int n = p.T * p.k;
    Routing r{-1, -1, 0.f, 0.f};
    if (lane < n) { r.e0 = __ldg(p.idx + lane); r.w0 = __ldg(p.wts + lane); }
    if (lane + 32 < n) { r.e1 = __ldg(p.idx + lane + 32); r.w1 = __ldg(p.wts + lane + 32); }
    return r;
}

// Union of routed experts over the T columns (one warp, T * k <= 64): slot 0
// is the shared expert (if any), then the distinct valid experts in ascending
// order.  An expert named twice in one column is one column of its slot; both
// entries point at it, so the combine adds its output once per entry (as the
// sum over j does).  An id out of range is dropped and flagged.
__device__ void build_slots(const MoeParams& p, SlotTable& S, const Routing& rt) {
    const int lane = threadIdx.x & 31;
    const int n = p.T * p.k;
    const int base = p.has_shared ? 1 : 0;
    // entry i is (column i / k, choice i % k); the quotient as a multiply-shift
    // (exact for i < 2^32 / k).  The passes below are loops of one copy with
    // the entry's slot kept in the table: this code runs once per launch, with
    // its instructions not yet in the cache.
    const uint32_t kdiv = 0xffffffffu / (uint32_t)p.k + 1u;
    S.mask[lane] = 0u;
    for (int s = lane; s < MOE_MAXS; s += 32) S.colmask[s] = 0u;
    __syncwarp();
#pragma unroll 1
    for (int i = lane; i < n; i += 32) {
        const int e = i < 32 ? rt.e0 : rt.e1;
        const int c = (int)__umulhi((uint32_t)i, kdiv), j = i - c * p.k;
        S.idx[i] = e;
        S.w[c][j] = i < 32 ? rt.w0 : rt.w1;
        S.tslot[c][j] = -1;
        if (e >= 0 && e < p.E) atomicOr(&S.mask[e >> 5], 1u << (e & 31));
        else set_error(p.ctrl, MOE_ERR_EXPERT);
    }
    __syncwarp();
    {
        const int pc = __popc(S.mask[lane]);
        int incl = pc;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        S.prefix[lane] = incl - pc;
        if (lane == 31) S.nslots = base + incl;
    }
    __syncwarp();
#pragma unroll 1
    for (int i = lane; i < n; i += 32) {
        const int e = S.idx[i];
        if (e < 0 || e >= p.E) continue;
        const int c = (int)__umulhi((uint32_t)i, kdiv), j = i - c * p.k;
        const int s = base + S.prefix[e >> 5] + __popc(S.mask[e >> 5] & ((1u << (e & 31)) - 1u));
        S.expert[s] = e;
        S.tslot[c][j] = (signed char)s;
        atomicOr(&S.colmask[s], 1u << c);
    }
    __syncwarp();
#pragma unroll 1
    for (int i = lane; i < n; i += 32) {
        const int c = (int)__umulhi((uint32_t)i, kdiv), j = i - c * p.k;
        const int s = S.tslot[c][j];
        if (s < 0) continue;
        const unsigned cm = S.colmask[s];
        const int pos = __popc(cm & ((1u << c) - 1u));   // columns ascend within a slot
        S.cols[s][pos] = (signed char)c;
        S.tpos[c][j] = (signed char)pos;
        if (pos == 0) S.ncols[s] = __popc(cm);   // several entries may write the same value
    }
    if (p.has_shared && lane == 0) {
        S.expert[0] = -1;
        S.ncols[0] = p.T;
        S.colmask[0] = (1u << p.T) - 1u;
        for (int c = 0; c < p.T; ++c) S.cols[0][c] = (signed char)c;
    }
    __syncwarp();
    // formats of every slot and the x copy of its gate/up tiles
    for (int s = lane; s < S.nslots; s += 32) {
        const int e = S.expert[s];
        int fa = p.fA, fb = p.fB;
        if (e < 0) { fa = p.fsA; fb = p.fsB; }
        else if (p.mix) { fa = __ldg(&p.mix[e].fa); fb = __ldg(&p.mix[e].fb); }
        S.fa[s] = (signed char)fa;
        S.fb[s] = (signed char)fb;
        S.ci[s] = (signed char)((p.nxc == 2 && p.xf[1] == fa) ? 1 : 0);
    }
    __syncwarp();
}

// Packed stream of the gate/up (phase 0) or down (phase 1) matrices of an
// expert (-1: the shared expert).
struct MatRef {
    const uint8_t* a;
    const uint8_t* b;
    int fmt;
};

__device__ __forceinline__ MatRef slot_mats(const MoeParams& p, int e, int ph) {
    if (ph == 0) {
        if (e < 0) return {p.shg, p.shu, p.fsA};
        if (p.mix) {
            const MoeMixEntry* m = p.mix + e;
            return {p.gate + __ldg(&m->og), p.up + __ldg(&m->ou), __ldg(&m->fa)};
        }
        return {p.gate + (long long)e * p.sg, p.up + (long long)e * p.su, p.fA};
    }
    if (e < 0) return {p.shd, nullptr, p.fsB};
    if (p.mix) return {p.down + __ldg(&p.mix[e].od), nullptr, __ldg(&p.mix[e].fb)};
    return {p.down + (long long)e * p.sd, nullptr, p.fB};
}

// ----------------------------------------------------------- work list ---
//
// Gate/up units (32 rows of I) u = slot * nrgA + i, u < nA, CTA u mod G.
// Down groups w = slot * ngB + j (row-groups 4j .. 4j + 3 of the slot, fewer
// at the slot's end), CTA (w - nA mod G) mod G.
constexpr int BGROUP = 4;
struct WorkList {
    int nrgA, nrgB, ngB, nA, nGB;
    __device__ void init(int nslots, int H, int I) {
        nrgA = I / 32;
        nrgB = (H + 15) / 16;
        ngB = (nrgB + BGROUP - 1) / BGROUP;
        nA = nslots * nrgA;
        nGB = nslots * ngB;
    }
};

// ------------------------------------------------------------- producer ---

struct ProdRing {
    int stage = 0, n = 0;
    uint32_t phase = 1;   // producer: parity to wait for on empty[stage] (fresh barriers pass)
};

__device__ __forceinline__ bool claim(const MoeParams& p, Shared& sh, ProdRing& rg) {
    return mbar_wait(&sh.empty[rg.stage], rg.phase, p.wait_limit);
}

__device__ __forceinline__ void advance(const MoeParams& p, ProdRing& rg) {
    ++rg.n;
    if (++rg.stage == p.ns) { rg.stage = 0; rg.phase ^= 1u; }
}

// Stages of one gate/up unit: its two row-groups, each in spans of up to 8
// chunks.
__device__ __forceinline__ int a_stages(int H) { return 2 * ((rfx_num_chunks(H) + MOE_CHUNKS_PER_STAGE - 1) / MOE_CHUNKS_PER_STAGE); }

// Stream stages [k0, k1) of gate/up unit `unit` of a slot (row-groups
// 2*unit and 2*unit + 1): one stage per span, one bulk copy per matrix (gate
// in the first half of the stage, up in the second).
__device__ bool issue_a(const MoeParams& p, Shared& sh, uint8_t* ring, ProdRing& q, int slot, int expert, int unit,
                        int k0, int k1, uint64_t pol, int& last_a) {
    const MatRef m = slot_mats(p, expert, 0);
    const int nch = rfx_num_chunks(p.H);
    const int nsp = (nch + MOE_CHUNKS_PER_STAGE - 1) / MOE_CHUNKS_PER_STAGE;
    const long long rgb = rfx_rowgroup_bytes(m.fmt, p.H);
    const int fullb = (int)rfx_chunk_bytes(m.fmt, 8);
    const uint32_t lastb = (uint32_t)rfx_chunk_bytes(m.fmt, rfx_chunk_tiles(p.H, nch - 1));
    for (int k = k0; k < k1; ++k) {
        const int hf = k / nsp, c0 = (k - hf * nsp) * MOE_CHUNKS_PER_STAGE;
        const int rg = 2 * unit + hf;
        const int c1 = min(nch, c0 + MOE_CHUNKS_PER_STAGE);
        const uint32_t bytes = (uint32_t)((c1 - 1 - c0) * fullb) + (c1 == nch ? lastb : (uint32_t)fullb);
        if (!claim(p, sh, q)) return false;
        StageRec r{};
        r.kind = 0;
        r.slot = (short)slot;
        r.rg = (short)rg;
        r.c0 = (short)c0;
        r.n = (short)hf;
        r.flags = (short)((c0 == 0 ? REC_FIRST : 0) | (c1 == nch ? REC_LAST : 0) | (c1 == nch && hf == 1 ? REC_CLOSE : 0));
        r.hbuf = -1;
        sh.rec[q.stage] = r;
        uint8_t* dst = ring + q.stage * MOE_STAGE_BYTES;
        const long long off = (long long)rg * rgb + (long long)c0 * fullb;
        mbar_arrive_expect_tx(&sh.full[q.stage], 2 * bytes);
        bulk_g2s(dst, m.a + off, bytes, &sh.full[q.stage], pol);
        bulk_g2s(dst + MOE_HALF_BYTES, m.b + off, bytes, &sh.full[q.stage], pol);
        last_a = q.n;
        advance(p, q);
    }
    return true;
}

// Bounded poll of a flag set by another CTA (acquire).
__device__ bool poll_flag(const uint32_t* f, uint32_t want, long long limit) {
    if (ld_acquire_gpu(f) >= want) return true;
    const long long t0 = clock64();
    unsigned nap = 32;
    while (ld_acquire_gpu(f) < want) {
        if (clock64() - t0 > limit) return false;
        __nanosleep(nap);
        nap = min(nap * 2u, 128u);
    }
    return true;
}

// Which slot's h image sits in which shared-memory buffer (the producer's view).
struct HState {
    int slot = -1;        // slot whose image is in buffer `buf`
    int buf = 1;          // the next image goes to buf ^ 1
    int copies[2] = {0, 0};
    bool announce = false;   // the next stage record carries REC_HNEW
};

// Make sure the h image of `slot` is in (or on its way to) a shared-memory
// buffer: wait until every gate/up unit of the slot has written its part of
// the image and the buffer is free, then one bulk copy.
__device__ bool ensure_h(const MoeParams& p, Shared& sh, uint8_t* xh, const ProdRing& q, HState& hs, int slot,
                         int ncols, int last_a, bool& x_drained) {
    if (hs.slot == slot) return true;
    const int b = hs.buf ^ 1;
    const int off = b ? p.hoff1 : p.hoff0;
    if (off < p.x_bytes && !x_drained) {
        // the buffer overlaps the staged x: every consumer must be past the
        // last gate/up stage (a later claim of its ring slot implies that)
        if (last_a >= 0 && q.n <= last_a + p.ns &&
            !mbar_wait(&sh.empty[last_a % p.ns], (uint32_t)(last_a / p.ns) & 1u, p.wait_limit))
            return false;
        x_drained = true;
    }
    if (!mbar_wait(&sh.hfree[b], ((uint32_t)hs.copies[b] & 1u) ^ 1u, p.wait_limit)) return false;
    if (!poll_flag(p.ctrl + MOE_CTRL_SLOT_DONE + slot, (uint32_t)(p.I / 32 + (p.fault == 2 ? 1 : 0)), p.wait_limit))
        return false;
    fence_proxy_async_global();   // generic-proxy writes of the image (another CTA) -> bulk-copy reads
    const uint32_t bytes = (uint32_t)moe_h_image_bytes(ncols, p.I);
    mbar_arrive_expect_tx(&sh.hfull[b], bytes);
    bulk_g2s(xh + off, p.hfrag + (long long)slot * p.hslot_bytes, bytes, &sh.hfull[b], policy_evict_last());
    ++hs.copies[b];
    hs.buf = b;
    hs.slot = slot;
    hs.announce = true;
    return true;
}

// Stream the down row-groups [u0, u0 + n): a stage holds two consecutive
// row-groups of one slot when a row-group fits one half (at most 8 chunks),
// else spans of 8 chunks.
__device__ __forceinline__ bool issue_b(const MoeParams& p, Shared& sh, uint8_t* ring, uint8_t* xh, ProdRing& q, HState& hs,
                        const WorkList& L, int u0, int n, uint64_t pol, int last_a, bool& x_drained) {
    const SlotTable& S = sh.st;
    const int nch = rfx_num_chunks(p.I);
    for (int u = u0; u < u0 + n;) {
        const int slot = u / L.nrgB, rg = u - slot * L.nrgB;
        if (!ensure_h(p, sh, xh, q, hs, slot, S.ncols[slot], last_a, x_drained)) return false;
        const MatRef m = slot_mats(p, S.expert[slot], 1);
        const long long rgb = rfx_rowgroup_bytes(m.fmt, p.I);
        if (nch <= MOE_CHUNKS_PER_STAGE) {
            const int pair = (u + 1 < u0 + n && (u + 1) / L.nrgB == slot) ? 2 : 1;
            if (!claim(p, sh, q)) return false;
            StageRec r{};
            r.kind = 1;
            r.slot = (short)slot;
            r.rg = (short)rg;
            r.c0 = 0;
            r.n = (short)pair;
            r.flags = (short)(REC_FIRST | REC_LAST | REC_CLOSE | (hs.announce ? REC_HNEW : 0));
            r.hbuf = (short)hs.buf;
            hs.announce = false;
            sh.rec[q.stage] = r;
            uint8_t* dst = ring + q.stage * MOE_STAGE_BYTES;
            mbar_arrive_expect_tx(&sh.full[q.stage], (uint32_t)(pair * rgb));
            for (int i = 0; i < pair; ++i)
                bulk_g2s(dst + i * MOE_HALF_BYTES, m.a + (long long)(rg + i) * rgb, (uint32_t)rgb, &sh.full[q.stage],
                         pol);
            advance(p, q);
            u += pair;
        } else {
            const int fullb = (int)rfx_chunk_bytes(m.fmt, 8);
            const uint32_t lastb = (uint32_t)rfx_chunk_bytes(m.fmt, rfx_chunk_tiles(p.I, nch - 1));
            for (int c0 = 0; c0 < nch; c0 += MOE_CHUNKS_PER_STAGE) {
                const int c1 = min(nch, c0 + MOE_CHUNKS_PER_STAGE);
                const uint32_t bytes = (uint32_t)((c1 - 1 - c0) * fullb) + (c1 == nch ? lastb : (uint32_t)fullb);
                if (!claim(p, sh, q)) return false;
                StageRec r{};
                r.kind = 1;
                r.slot = (short)slot;
                r.rg = (short)rg;
                r.c0 = (short)c0;
                r.n = 1;
                r.flags = (short)((c0 == 0 ? REC_FIRST : 0) | (c1 == nch ? REC_LAST | REC_CLOSE : 0) |
                                  (hs.announce ? REC_HNEW : 0));
                r.hbuf = (short)hs.buf;
                hs.announce = false;
                sh.rec[q.stage] = r;
                uint8_t* dst = ring + q.stage * MOE_STAGE_BYTES;
                mbar_arrive_expect_tx(&sh.full[q.stage], bytes);
                bulk_g2s(dst, m.a + (long long)rg * rgb + (long long)c0 * fullb, bytes, &sh.full[q.stage], pol);
                advance(p, q);
            }
            ++u;
        }
    }
    return true;
}

// The producer lane after the routing is known: this CTA's gate/up units
// (the first `pre` stages of the first were streamed before the wait), then
// its down groups.
__device__ void producer(const MoeParams& p, Shared& sh, uint8_t* ring, uint8_t* xh, ProdRing& q, int pre,
                         int last_a) {
    const SlotTable& S = sh.st;
    const int G = gridDim.x;
    WorkList L;
    L.init(S.nslots, p.H, p.I);
    const uint64_t pol = policy_evict_first();
    HState hs;
    bool x_drained = false;
    bool ok = true;
    const int nst = a_stages(p.H);
    for (int u = (int)blockIdx.x; ok && u < L.nA; u += G) {
        const int slot = u / L.nrgA, i = u - slot * L.nrgA;
        ok = issue_a(p, sh, ring, q, slot, S.expert[slot], i, u == (int)blockIdx.x ? pre : 0, nst, pol, last_a);
    }
    const int w0 = ((int)blockIdx.x - L.nA % G + G) % G;
    for (int w = w0; ok && w < L.nGB; w += G) {
        const int slot = w / L.ngB, j = w - slot * L.ngB;
        const int u0 = slot * L.nrgB + BGROUP * j;
        ok = issue_b(p, sh, ring, xh, q, hs, L, u0, min(BGROUP, L.nrgB - BGROUP * j), pol, last_a, x_drained);
    }
    // end-of-work record: a stage with no copy
    if (ok) {
        if (claim(p, sh, q)) {
            StageRec r{};
            r.kind = -1;
            r.flags = REC_END;
            sh.rec[q.stage] = r;
            mbar_arrive(&sh.full[q.stage]);
            advance(p, q);
        } else {
            ok = false;
        }
    }
    if (!ok) {
        set_error(p.ctrl, MOE_ERR_TIMEOUT);
        sh.abort_flag = 1;
        // tell the consumers to stop (if a stage can still be claimed), then
        // wait (bounded) until every issued copy has landed
        if (mbar_wait(&sh.empty[q.stage], q.phase, p.wait_limit)) {
            StageRec r{};
            r.kind = -1;
            r.flags = REC_END;
            sh.rec[q.stage] = r;
            mbar_arrive(&sh.full[q.stage]);
            advance(p, q);
        }
        for (int i = sh.consumed; i < q.n; ++i) (void)mbar_wait(&sh.full[i % p.ns], (i / p.ns) & 1, p.wait_limit);
        for (int b = 0; b < 2; ++b)
            if (hs.copies[b]) (void)mbar_wait(&sh.hfull[b], (uint32_t)(hs.copies[b] - 1) & 1u, p.wait_limit);
    }
}

// ----------------------------------------------------------- grid barrier ---
//
// One thread per CTA: a release add on a 64-bit counter that only grows, then
// an acquire poll until every CTA of this launch has added.  The target is the
// next multiple of the grid size above the value this CTA saw, so the counter
// needs no reset between calls (a timed-out call leaves it unaligned: the
// workspace must then be re-initialised).  Returns false on timeout.
__device__ bool grid_barrier(unsigned long long* ctr, long long limit, int extra) {
    const unsigned long long G = gridDim.x;
    const unsigned long long old = atom_add_release_gpu_u64(ctr, 1ull);
    const unsigned long long target = (old / G + 1) * G + (unsigned long long)extra;
    const long long t0 = clock64();
    unsigned nap = 32;
    while (ld_acquire_gpu_u64(ctr) < target) {
        if (clock64() - t0 > limit) return false;
        __nanosleep(nap);
        nap = min(nap * 2u, 256u);
    }
    return true;
}

// ------------------------------------------------------------- epilogues ---

// A reduction buffer holds the 8 consumer warps' partials of up to two
// row-groups (half h at h * moe_red_bytes(QC)).  In a half, lane (g, t) =
// (lane >> 2, lane & 3) of a warp holds rows g, g+8 and columns 2t, 2t+1
// (gate/up: gate then up; down: the hi/lo virtual columns of real column t,
// then of t + 4).  Only lanes that can hold a live column store:
//   T = 1:   lanes t = 0, one float4 (gate g, g+8, up g, g+8 / hi g, lo g,
//            hi g+8, lo g+8) at [warp][g];
//   T <= 4:  gate/up: lanes t < 2, [warp][half][2g + t][4]; down: every lane,
//            [warp][lane][4];
//   T <= 8:  every lane, [warp][half][lane][4].
// The epilogue sums the 8 warps in warp order.
template <int QC>
__device__ __forceinline__ void red_store(uint8_t* buf, int w, int lane, bool unit_a, const float v[8]) {
    const int g = lane >> 2, t = lane & 3;
    if constexpr (QC == 1) {
        uint8_t* my = buf + w * 128 + g * 16;
        if (t == 0) {
            if (unit_a) *reinterpret_cast<float4*>(my) = make_float4(v[0], v[2], v[4], v[6]);
            else *reinterpret_cast<float4*>(my) = make_float4(v[0], v[1], v[2], v[3]);
        }
    } else if constexpr (QC == 2) {
        uint8_t* my = buf + w * 512;
        if (unit_a) {
            if (t < 2) {
                *reinterpret_cast<float4*>(my + (2 * g + t) * 16) = make_float4(v[0], v[1], v[2], v[3]);
                *reinterpret_cast<float4*>(my + 256 + (2 * g + t) * 16) = make_float4(v[4], v[5], v[6], v[7]);
            }
        } else {
            *reinterpret_cast<float4*>(my + lane * 16) = make_float4(v[0], v[1], v[2], v[3]);
        }
    } else {
        uint8_t* my = buf + w * 1024;
        *reinterpret_cast<float4*>(my + lane * 16) = make_float4(v[0], v[1], v[2], v[3]);
        *reinterpret_cast<float4*>(my + 512 + lane * 16) = make_float4(v[4], v[5], v[6], v[7]);
    }
}

// Sum of the 8 warps' partials of one half for this lane's (g, t), warp
// order; lanes without a live column get zeros.  a: gate (or down n-block 0),
// b: up (or down n-block 1).
template <int QC>
__device__ __forceinline__ void red_sum(const uint8_t* buf, int lane, bool unit_a, float a[4], float b[4]) {
    const int g = lane >> 2, t = lane & 3;
    float4 s0 = make_float4(0.f, 0.f, 0.f, 0.f), s1 = s0;
    if constexpr (QC == 1) {
        if (t == 0) {
#pragma unroll
            for (int w = 0; w < NCW; ++w) {
                const float4 v = ldsf4(buf + w * 128 + g * 16);
                s0.x += v.x; s0.y += v.y; s0.z += v.z; s0.w += v.w;
            }
        }
        if (unit_a) {   // (gate g, gate g+8, up g, up g+8) -> acc order (g c0, g c1, g+8 c0, g+8 c1)
            a[0] = s0.x; a[1] = 0.f; a[2] = s0.y; a[3] = 0.f;
            b[0] = s0.z; b[1] = 0.f; b[2] = s0.w; b[3] = 0.f;
        } else {
            a[0] = s0.x; a[1] = s0.y; a[2] = s0.z; a[3] = s0.w;
            b[0] = b[1] = b[2] = b[3] = 0.f;
        }
        return;
    } else if constexpr (QC == 2) {
        if (unit_a) {
            if (t < 2) {
#pragma unroll
                for (int w = 0; w < NCW; ++w) {
                    const float4 x = ldsf4(buf + w * 512 + (2 * g + t) * 16);
                    const float4 y = ldsf4(buf + w * 512 + 256 + (2 * g + t) * 16);
                    s0.x += x.x; s0.y += x.y; s0.z += x.z; s0.w += x.w;
                    s1.x += y.x; s1.y += y.y; s1.z += y.z; s1.w += y.w;
                }
            }
        } else {
#pragma unroll
            for (int w = 0; w < NCW; ++w) {
                const float4 x = ldsf4(buf + w * 512 + lane * 16);
                s0.x += x.x; s0.y += x.y; s0.z += x.z; s0.w += x.w;
            }
        }
    } else {
#pragma unroll
        for (int w = 0; w < NCW; ++w) {
            const float4 x = ldsf4(buf + w * 1024 + lane * 16);
            const float4 y = ldsf4(buf + w * 1024 + 512 + lane * 16);
            s0.x += x.x; s0.y += x.y; s0.z += x.z; s0.w += x.w;
            s1.x += y.x; s1.y += y.y; s1.z += y.z; s1.w += y.w;
        }
    }
    a[0] = s0.x; a[1] = s0.y; a[2] = s0.z; a[3] = s0.w;
    b[0] = s1.x; b[1] = s1.y; b[2] = s1.z; b[3] = s1.w;
}

// 2^e as a product of two normal powers of two (|e| <= 250).
__device__ __forceinline__ void pow2_pair(int e, float& f1, float& f2) {
    f1 = __int_as_float((127 + e / 2) << 23);
    f2 = __int_as_float((127 + e - e / 2) << 23);
}

// A gate/up unit (row-groups rg0, rg0 + 1 = 32 values of I): undo the
// per-column x scaling, h = silu(g) * u, then the slot's h image for these 32
// values: per column the exponent n (max |h| * 2^n in [2^14, 2^15)), the
// fp16 hi/lo pair of h * 2^n at the down projection's B-fragment positions
// ([step][virtual column 2*col + {0 hi, 1 lo}][t][4]: rows 2t, 2t+1, 2t+8,
// 2t+9 of the step), each 16-row step's sum of (hi + lo) and 2^-n.  Lane
// (g, t) holds rows g, g+8 of both steps for columns 2t, 2t+1; after one
// exchange with lane ^ 4, even-g lanes write column 2t and odd-g lanes column
// 2t+1 as 8-byte pieces.
template <int QC>
__device__ void epilogue_a(const MoeParams& p, Shared& sh, const uint8_t* rb, int slot, int ncols, int rg0,
                           int lane) {
    const int g = lane >> 2, t = lane & 3;
    const int RB = moe_red_bytes(QC);
    constexpr bool C1 = QC >= 2;   // the lane's second column (2t + 1) can be live
    float h[2][4];
    float m[2] = {0.f, 0.f};
    bool bad = false;
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
        float G[4], U[4];
        red_sum<QC>(rb + hf * RB, lane, true, G, U);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int col = 2 * t + (i & 1);
            float hv = 0.f;
            if ((C1 || !(i & 1)) && col < ncols) {
                const float sc = __int_as_float((127 - sh.xn[sh.st.cols[slot][col]]) << 23);
                const float gv = G[i] * sc, uv = U[i] * sc;
                hv = gv >= -64.f ? gv / (1.0f + expf(-gv)) * uv : silu_mul_tail(gv, uv);
                if (!isfinite(hv)) bad = true;
            }
            h[hf][i] = hv;
            m[i & 1] = fmaxf(m[i & 1], fabsf(hv));
        }
    }
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
        m[0] = fmaxf(m[0], __shfl_xor_sync(0xffffffffu, m[0], o));
        m[1] = fmaxf(m[1], __shfl_xor_sync(0xffffffffu, m[1], o));
    }
    float up1[2], up2[2], dn[2];
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const uint32_t mb = __float_as_uint(m[j]);
        const int ex = (int)((mb >> 23) & 255u);
        int n = (mb == 0u || ex == 255) ? 0 : 14 - (ex - 127);
        n = max(-250, min(250, n));
        pow2_pair(n, up1[j], up2[j]);
        float d1, d2;
        pow2_pair(-n, d1, d2);
        dn[j] = d1 * d2;   // 2^-n, normal for |n| <= 126; a subnormal or zero factor otherwise
    }
    uint32_t pk[2][4];
    float sum[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
#pragma unroll
    for (int hf = 0; hf < 2; ++hf)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float a = h[hf][i] * up1[i & 1] * up2[i & 1];
            const __half hi = __float2half_rn(a);
            const __half lo = __float2half_rn(a - __half2float(hi));
            pk[hf][i] = (uint32_t)__half_as_ushort(hi) | ((uint32_t)__half_as_ushort(lo) << 16);
            sum[hf][i & 1] += __half2float(hi) + __half2float(lo);
        }
    uint8_t* img = p.hfrag + (long long)slot * p.hslot_bytes;
    float* hsum = reinterpret_cast<float*>(img + 4 * ncols * p.I);
    float* hsc = hsum + ncols * moe_sstr(p.I);
    const bool ev = (g & 1) == 0;
    const int colw = 2 * t + (g & 1);
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
        const uint32_t ra = __shfl_xor_sync(0xffffffffu, ev ? pk[hf][1] : pk[hf][0], 4);
        const uint32_t rb2 = __shfl_xor_sync(0xffffffffu, ev ? pk[hf][3] : pk[hf][2], 4);
        const uint32_t q0 = ev ? pk[hf][0] : ra, q1 = ev ? ra : pk[hf][1];
        const uint32_t q2 = ev ? pk[hf][2] : rb2, q3 = ev ? rb2 : pk[hf][3];
        if (colw < ncols) {
            uint2 hi2, lo2;
            hi2.x = (q0 & 0xffffu) | (q1 << 16);
            hi2.y = (q2 & 0xffffu) | (q3 << 16);
            lo2.x = (q0 >> 16) | (q1 & 0xffff0000u);
            lo2.y = (q2 >> 16) | (q3 & 0xffff0000u);
            uint8_t* dst = img + ((long long)((rg0 + hf) * 2 * ncols + 2 * colw) * 4 + (g >> 1)) * 8;
            *reinterpret_cast<uint2*>(dst) = hi2;
            *reinterpret_cast<uint2*>(dst + 32) = lo2;
        }
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
            sum[hf][0] += __shfl_xor_sync(0xffffffffu, sum[hf][0], o);
            sum[hf][1] += __shfl_xor_sync(0xffffffffu, sum[hf][1], o);
        }
    }
    if (g == 0) {
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int col = 2 * t + j;
            if (col < ncols) {
                hsum[col * moe_sstr(p.I) + rg0] = sum[0][j];
                hsum[col * moe_sstr(p.I) + rg0 + 1] = sum[1][j];
                hsc[col * moe_sbs(p.I) + rg0 / 2] = dn[j];
            }
        }
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) set_error(p.ctrl, MOE_ERR_RANGE);
}

// Partial down outputs of the n row-groups of a unit -> dpart[slot][col][rows].
template <int QC>
__device__ void epilogue_b(const MoeParams& p, const uint8_t* rb, int slot, int ncols, int rg, int n, int lane) {
    const int g = lane >> 2, t = lane & 3;
    float* dp = p.dpart + (long long)slot * p.T * p.H;
    constexpr int NB = QC == 3 ? 2 : 1;
    for (int hf = 0; hf < n; ++hf) {
        float D[8];
        red_sum<QC>(rb + hf * moe_red_bytes(QC), lane, false, D, D + 4);
        const int row0 = 16 * (rg + hf) + g;
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) {
            const int col = 4 * nb + t;  // virtual columns 2col (hi), 2col+1 (lo)
            if (col < ncols && (QC != 1 || t == 0)) {
                dp[(long long)col * p.H + row0] = D[4 * nb + 0] + D[4 * nb + 1];
                dp[(long long)col * p.H + row0 + 8] = D[4 * nb + 2] + D[4 * nb + 3];
            }
        }
    }
}

// Count gate/up units done: one fence orders all the warp's stores so far
// (lane 0 is ordered after the other lanes' stores by the warp barrier), then
// one release reduction per unit.
__device__ __forceinline__ void flush_done(const MoeParams& p, int lane, int& npend, const int* pend) {
    __syncwarp();
    if (npend && lane == 0) {
        __threadfence();
        for (int i = 0; i < npend; ++i) red_add_release_gpu(p.ctrl + MOE_CTRL_SLOT_DONE + pend[i], 1u);
    }
    npend = 0;
}

// An epilogue warp: units r = e, e + NEPI, ... in the order the consumers
// deposit them.  The done counts of gate/up units are published when the next
// unit is not there yet (the fence then costs no throughput), or after 2.
template <int QC>
__device__ void epilogue_warp(const MoeParams& p, Shared& sh, uint8_t* red, int e) {
    const int lane = threadIdx.x & 31;
    int pend[2];
    int npend = 0;
    for (int r = e;; r += NEPI) {
        const int b = r % p.nred;
        const uint32_t ph = (uint32_t)(r / p.nred) & 1u;
        if (npend && (npend == 2 || !mbar_test_wait(&sh.rfull[b], ph))) flush_done(p, lane, npend, pend);
        if (!mbar_wait(&sh.rfull[b], ph, p.wait_limit)) {
            if (lane == 0) { set_error(p.ctrl, MOE_ERR_TIMEOUT); sh.abort_flag = 1; }
            break;
        }
        const RedInfo ri = sh.rinfo[b];
        if (ri.kind == UNIT_END) break;
        const uint8_t* rb = red + b * 2 * moe_red_bytes(QC);
        if (ri.kind == UNIT_A) {
            epilogue_a<QC>(p, sh, rb, ri.slot, ri.ncols, ri.rg, lane);
            pend[npend++] = ri.slot;
        } else {
            epilogue_b<QC>(p, rb, ri.slot, ri.ncols, ri.rg, ri.n, lane);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.rempty[b]);
    }
    flush_done(p, lane, npend, pend);
}

// ------------------------------------------------------------- consumers ---

struct RedCursor {
    int b = 0;
    uint32_t ph = 0;   // parity of the rfull phase being filled; rempty waits for ph ^ 1
};

// Deposit this warp's partials of one row-group into half `half` of the
// current reduction buffer (waiting for the buffer at half 0); `close` hands
// the unit to its epilogue warp.
template <int QC>
__device__ __forceinline__ bool red_deposit(const MoeParams& p, Shared& sh, uint8_t* red, RedCursor& rc, int w,
                                            int lane, const float v[8], int half, bool close, const RedInfo& info) {
    if (half == 0 && !mbar_wait(&sh.rempty[rc.b], rc.ph ^ 1u, p.wait_limit)) return false;
    red_store<QC>(red + (2 * rc.b + half) * moe_red_bytes(QC), w, lane, info.kind == UNIT_A, v);
    if (close) {
        if (w == 0 && lane == 0) sh.rinfo[rc.b] = info;
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.rfull[rc.b]);
        if (++rc.b == p.nred) { rc.b = 0; rc.ph ^= 1u; }
    }
    return true;
}

// Bit offset of tile (k/32) of a K-long row-group for format fmt (0 inside a
// trailing partial chunk, which is decoded to exact levels).
__device__ __forceinline__ int s_pos(int fmt, int k, int K) {
    const int blk = k >> 5;
    if ((blk >> 3) == (K >> 8) && (K & 255)) return 0;
    const int b = blk & 7;
    return fmt == 2 ? Plane<2>::s_of(b) : (fmt == 3 ? Plane<3>::s_of(b) : Plane<4>::s_of(b));
}

__device__ __forceinline__ void ld8(const float* src, float d[8]) {
    const float4 a = ldsf4((const uint8_t*)src), b = ldsf4((const uint8_t*)(src + 4));
    d[0] = a.x; d[1] = a.y; d[2] = a.z; d[3] = a.w;
    d[4] = b.x; d[5] = b.y; d[6] = b.z; d[7] = b.w;
}

// One gate/up chunk pair (chunk c of the stage's span, this warp's share).
template <int FMT, int FC, bool TWO, class SRC>
__device__ __forceinline__ void stepA(const uint8_t* st, int c, int H, int lane, int g, const SRC& bs, const float* sA0,
                                      const float* sA1, AccA& ag, AccA& au) {
    const int nt = rfx_chunk_tiles(H, c);
    if (nt == 8) {
        float S0[8], S1[8];
        ld8(sA0 + 8 * c, S0);
        if (TWO) ld8(sA1 + 8 * c, S1);
        chunkA_full<FMT, FC, TWO>(st, st + MOE_HALF_BYTES, lane, g, bs, c * 16, S0, S1, ag, au);
    } else {
        chunkA_partial<FMT, true>(st, st + MOE_HALF_BYTES, nt, lane, g, bs, c * 16, ag, au);
    }
}

// One down chunk.  hsc: the image's 2^-n factors [ncols][sbs].
template <int FMT, int NB, class SRC>
__device__ __forceinline__ void stepB(const uint8_t* st, int c, int I, int lane, int g, int t, const SRC* bs,
                                      const float* hsum, const float* hsc, int ncols, int sstr, int sbs, AccB<NB>& ab) {
    const int nt = rfx_chunk_tiles(I, c);
    float Hs[NB][8];
#pragma unroll
    for (int nb = 0; nb < NB; ++nb) {
        const int colr = 4 * nb + t;
        const float* hp = hsc + (colr < ncols ? colr : 0) * sbs + 8 * c;
        const float4 a = ldsf4((const uint8_t*)hp), b = ldsf4((const uint8_t*)(hp + 4));
        Hs[nb][0] = a.x; Hs[nb][1] = a.y; Hs[nb][2] = a.z; Hs[nb][3] = a.w;
        Hs[nb][4] = b.x; Hs[nb][5] = b.y; Hs[nb][6] = b.z; Hs[nb][7] = b.w;
    }
    if (nt == 8) {
        // block sums of h for the lane's real column(s): two halves per block
        float Sb[NB][8];
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) {
            const int colr = 4 * nb + t;
            const float* hp = hsum + (colr < ncols ? colr : 0) * sstr + 16 * c;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float4 x4 = ldsf4((const uint8_t*)(hp + 4 * q));
                Sb[nb][2 * q] = x4.x + x4.y;
                Sb[nb][2 * q + 1] = x4.z + x4.w;
            }
        }
        chunkB_full<FMT, NB>(st, lane, g, bs, c * 16, Sb, Hs, ab);
    } else {
        chunkB_partial<FMT, NB>(st, nt, lane, g, bs, c * 16, Hs, ab);
    }
}

// A consumer warp's ring cursor.
struct ConsRing {
    int stage = 0, cc = 0;
    uint32_t phase = 0;
};

__device__ __forceinline__ void cons_release(const MoeParams& p, Shared& sh, ConsRing& rp, int w, int lane) {
    __syncwarp();
    if (lane == 0) mbar_arrive(&sh.empty[rp.stage]);
    ++rp.cc;
    if (w == 0 && lane == 0) sh.consumed = rp.cc;
    if (++rp.stage == p.ns) { rp.stage = 0; rp.phase ^= 1u; }
}

__device__ __forceinline__ bool cons_next(const MoeParams& p, Shared& sh, ConsRing& rp, StageRec& r) {
    if (!mbar_wait(&sh.full[rp.stage], rp.phase, p.wait_limit)) return false;
    r = sh.rec[rp.stage];
    return true;
}

// Gate/up loop variant of a slot: 8 * its format + the format of its x copy
// (when they differ, the scales carry the difference of the bit offsets).
__device__ __forceinline__ int variant_a(const MoeParams& p, const SlotTable& S, int slot) {
    return 8 * S.fa[slot] + p.xf[S.ci[slot]];
}
__device__ __forceinline__ int fmt_b(const SlotTable& S, int slot) { return S.fb[slot]; }

// Gate/up stages of one variant (format FMT, x copy of format FC), from the
// current record r (first span of a row-group) while the records stay gate/up
// spans of that variant; returns with the next record in r.
template <int FMT, int FC, bool TWO, int QC>
__device__ __forceinline__ bool loop_a(const MoeParams& p, Shared& sh, uint8_t* ring, uint8_t* xh, uint8_t* red,
                                       ConsRing& rp, RedCursor& rc, StageRec& r) {
    const SlotTable& S = sh.st;
    const int w = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int nxc = p.nxc;
    const float* sx = (const float*)(xh + nxc * p.T * p.x_stride);   // [copy][col][sxs]
    const int sxs = moe_sxs(p.H);
    const int nch = rfx_num_chunks(p.H);
    constexpr int FULLB = 128 * (FMT * 4 + (FMT == 4 ? 1 : 2));
    AccA ag, au;
    BSrcK<32> bs{xh, 0};
    const float* sA0 = sx;
    const float* sA1 = sx;
    int slot = 0, ncols = 1;
    while (true) {
        if (r.flags & REC_FIRST) {
            slot = r.slot;
            ncols = S.ncols[slot];
            const int ci = S.ci[slot];
            const int colg = S.cols[slot][g < ncols ? g : 0];
            bs.base = xh + (ci * p.T + colg) * p.x_stride + t * 8;
            const int c0 = S.cols[slot][2 * t < ncols ? 2 * t : 0];
            const int c1 = S.cols[slot][2 * t + 1 < ncols ? 2 * t + 1 : 0];
            sA0 = sx + (ci * p.T + c0) * sxs;
            sA1 = sx + (ci * p.T + c1) * sxs;
            ag.zero();
            au.zero();
        }
        const int c = r.c0 + w;
        if (c < nch)
            stepA<FMT, FC, TWO>(ring + rp.stage * MOE_STAGE_BYTES + w * FULLB, c, p.H, lane, g, bs, sA0, sA1, ag, au);
        cons_release(p, sh, rp, w, lane);
        if (r.flags & REC_LAST) {
            float v[8];
            finishA<FMT>(ag, v);
            finishA<FMT>(au, v + 4);
            if (!red_deposit<QC>(p, sh, red, rc, w, lane, v, r.n, (r.flags & REC_CLOSE) != 0,
                                 RedInfo{UNIT_A, slot, ncols, r.rg - r.n, 2}))
                return false;
        }
        if (!cons_next(p, sh, rp, r)) return false;
        if (r.kind != 0 || ((r.flags & REC_FIRST) && variant_a(p, S, r.slot) != 8 * FMT + FC)) return true;
    }
}

// The variants whose x copy is of another format: ROCmFPX MIX layers with a
// gate/up format that has no copy of its own (a kernel of their own, so that
// the common variants keep their register allocation).
template <bool TWO, int QC>
__device__ __forceinline__ bool loop_a_other(const MoeParams& p, Shared& sh, uint8_t* ring, uint8_t* xh, uint8_t* red,
                                             ConsRing& rp, RedCursor& rc, StageRec& r, int v) {
    switch (v) {
        case 8 * 2 + 3: return loop_a<2, 3, TWO, QC>(p, sh, ring, xh, red, rp, rc, r);
        case 8 * 2 + 4: return loop_a<2, 4, TWO, QC>(p, sh, ring, xh, red, rp, rc, r);
        case 8 * 3 + 2: return loop_a<3, 2, TWO, QC>(p, sh, ring, xh, red, rp, rc, r);
        case 8 * 3 + 4: return loop_a<3, 4, TWO, QC>(p, sh, ring, xh, red, rp, rc, r);
        case 8 * 4 + 2: return loop_a<4, 2, TWO, QC>(p, sh, ring, xh, red, rp, rc, r);
        case 8 * 4 + 3: return loop_a<4, 3, TWO, QC>(p, sh, ring, xh, red, rp, rc, r);
        default: return false;
    }
}

// The consumers' view of the slot whose h image is in use.
template <int NB, int HSTRIDE>
struct HView {
    BSrcK<HSTRIDE> bs[NB];
    const float* hsum;
    const float* hsc;
    int slot = -1, ncols = 1;
    int cur = -1;      // buffer in use
    int cnt[2] = {0, 0};
};

// Down stages of one format (one or two row-groups per stage, see the
// producer), from the current record r while the records stay down spans of
// that format; returns with the next record in r.
template <int FMT, int NB, int HSTRIDE, int QC>
__device__ __forceinline__ bool loop_b(const MoeParams& p, Shared& sh, uint8_t* ring, uint8_t* xh, uint8_t* red,
                                       ConsRing& rp, RedCursor& rc, StageRec& r, HView<NB, HSTRIDE>& hv) {
    const SlotTable& S = sh.st;
    const int w = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int nch = rfx_num_chunks(p.I);
    const int sstr = moe_sstr(p.I), sbs = moe_sbs(p.I);
    constexpr int FULLB = 128 * (FMT * 4 + (FMT == 4 ? 1 : 2));
    AccB<NB> ab;
    while (true) {
        if (r.flags & REC_HNEW) {
            const int b = r.hbuf;
            if (!mbar_wait(&sh.hfull[b], (uint32_t)hv.cnt[b] & 1u, p.wait_limit)) return false;
            ++hv.cnt[b];
            if (hv.cur >= 0 && hv.cur != b) {
                __syncwarp();
                if (lane == 0) mbar_arrive(&sh.hfree[hv.cur]);
            }
            hv.cur = b;
            hv.slot = r.slot;
            hv.ncols = S.ncols[r.slot];
            const uint8_t* img = xh + (b ? p.hoff1 : p.hoff0);
            const int vst = 64 * hv.ncols;  // bytes per k16 step
#pragma unroll
            for (int nb = 0; nb < NB; ++nb) {
                const int vv = min(8 * nb + g, 2 * hv.ncols - 1);
                hv.bs[nb] = BSrcK<HSTRIDE>{img + (vv * 4 + t) * 8, vst};
            }
            hv.hsum = (const float*)(img + 4 * hv.ncols * p.I);
            hv.hsc = hv.hsum + hv.ncols * sstr;
        }
        const int c = r.c0 + w;
        // the stage's row-groups one after the other (one copy of the chunk code)
#pragma unroll 1
        for (int i = 0; i < r.n; ++i) {
            if (r.flags & REC_FIRST) ab.zero();
            if (c < nch)
                stepB<FMT, NB>(ring + rp.stage * MOE_STAGE_BYTES + i * MOE_HALF_BYTES + w * FULLB, c, p.I, lane, g, t,
                               hv.bs, hv.hsum, hv.hsc, hv.ncols, sstr, sbs, ab);
            if (r.flags & REC_LAST) {
                float vb[NB][4], v[8];
                finishB<FMT, NB>(ab, vb);
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    v[k] = vb[0][k];
                    v[4 + k] = NB > 1 ? vb[NB - 1][k] : 0.f;
                }
                if (!red_deposit<QC>(p, sh, red, rc, w, lane, v, i, i == r.n - 1 && (r.flags & REC_CLOSE) != 0,
                                     RedInfo{UNIT_B, hv.slot, hv.ncols, r.rg, r.n}))
                    return false;
            }
        }
        cons_release(p, sh, rp, w, lane);
        if (!cons_next(p, sh, rp, r)) return false;
        if (r.kind != 1 || fmt_b(S, r.slot) != FMT) return true;
    }
}

// Consumer warp: the records of a CTA's stream are its gate/up spans, then its
// down spans, then the end record.  Each phase runs one loop per format.
template <int QC, bool OTHER>
__device__ void consumer(const MoeParams& p, Shared& sh, uint8_t* ring, uint8_t* xh, uint8_t* red) {
    constexpr bool TWO = QC >= 2;           // a second live column per lane in the gate/up output
    constexpr int NB = QC >= 3 ? 2 : 1;     // n-blocks of virtual (hi, lo) columns in the down projection
    constexpr int HSTRIDE = QC == 1 ? 64 : 0;   // bytes per k16 step of h (one column: 2 virtual x 4 lanes x 8 B)
    const SlotTable& S = sh.st;
    const int w = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    ConsRing rp;
    RedCursor rc;
    StageRec r{};
    HView<NB, HSTRIDE> hv;
    bool ok = cons_next(p, sh, rp, r);
    while (ok && r.kind == 0) {
        const int v = variant_a(p, S, r.slot);
        if (v == 8 * 2 + 2) ok = loop_a<2, 2, TWO, QC>(p, sh, ring, xh, red, rp, rc, r);
        else if (v == 8 * 3 + 3) ok = loop_a<3, 3, TWO, QC>(p, sh, ring, xh, red, rp, rc, r);
        else if (v == 8 * 4 + 4) ok = loop_a<4, 4, TWO, QC>(p, sh, ring, xh, red, rp, rc, r);
        else if constexpr (OTHER) ok = loop_a_other<TWO, QC>(p, sh, ring, xh, red, rp, rc, r, v);
        else ok = false;
    }
    while (ok && r.kind == 1) {
        const int f = fmt_b(S, r.slot);
        if (f == 3) ok = loop_b<3, NB, HSTRIDE, QC>(p, sh, ring, xh, red, rp, rc, r, hv);
        else if (f == 2) ok = loop_b<2, NB, HSTRIDE, QC>(p, sh, ring, xh, red, rp, rc, r, hv);
        else ok = loop_b<4, NB, HSTRIDE, QC>(p, sh, ring, xh, red, rp, rc, r, hv);
    }
    if (ok && r.kind >= 0) ok = false;   // a record of an unexpected kind
    if (ok) cons_release(p, sh, rp, w, lane);   // the end record's stage
    if (!ok && lane == 0) {
        set_error(p.ctrl, MOE_ERR_TIMEOUT);
        sh.abort_flag = 1;
    }
    // one end-of-work unit for each epilogue warp
    const float z[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int i = 0; i < NEPI; ++i) (void)red_deposit<QC>(p, sh, red, rc, w, lane, z, 0, true, RedInfo{UNIT_END, 0, 0, 0, 0});
}

// x (bf16 [T][H], global) -> shared memory for the gate/up B operand: per
// column c, x * 2^xn[c] with xn[c] putting max|x| in [2^13, 2^14), times
// 2^-s_b for the tile's bit offset in the gate/up format (one copy per format
// in use), rounded to fp16 in fragment order [c][step][t][k 2t,2t+1,2t+8,2t+9];
// plus the block sums of the staged values (times 2^s_b) for the offset
// correction.  Run by `nthr` threads (sid = 0 .. nthr-1, whole warps).  An
// item is 8 consecutive values of a column (one 16-byte load), item i =
// c * H/8 + j; thread sid takes items sid, sid + nthr, ...; 4 consecutive
// items (4 consecutive lanes) are one 32-block.  Each round issues all of a
// thread's loads (up to XR items) before using any.
constexpr int XR = 8;

// Column of item i: i / per_col as a multiply and shift, with
// cdiv = floor(2^32 / per_col) + 1 (exact while i * per_col < 2^32; here
// i < MOE_MAXT * per_col and per_col = H / 8).
__device__ __forceinline__ int x_col(int i, uint32_t cdiv) { return (int)__umulhi((uint32_t)i, cdiv); }

// Max |x| of one item per column into sh.xmax (one shared atomic per column
// the warp's items touch; i0 = the warp's first item, warp-uniform).
__device__ __forceinline__ void x_max(Shared& sh, const uint4& v, int i0, int lane, int nitems, uint32_t cdiv) {
    const int i = i0 + lane;
    const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
    uint32_t m = 0u;
#pragma unroll
    for (int e = 0; e < 4; ++e) m = max(m, max((wv[e] << 16) & 0x7fffffffu, wv[e] & 0x7fff0000u));
    const int cmine = i < nitems ? x_col(i, cdiv) : -1;
    const int ca = x_col(i0, cdiv), cb = x_col(min(i0 + 31, nitems - 1), cdiv);
#pragma unroll 1
    for (int c = ca; c <= cb; ++c) {
        const uint32_t mc = __reduce_max_sync(0xffffffffu, cmine == c ? m : 0u);
        if (lane == 0 && mc) atomicMax(&sh.xmax[c], mc);
    }
}

// Scaled fp16 fragments and block sums of one item, for every gate/up format copy.
__device__ __forceinline__ void x_put(const MoeParams& p, Shared& sh, uint8_t* xh, float* sx, int sxs, int nxc,
                                      const uint4& v, int i0, int lane, int nitems, int per_col, uint32_t cdiv) {
    const int i = i0 + lane;
    const bool in = i < nitems;
    const int c = in ? x_col(i, cdiv) : 0, j = in ? i - c * per_col : 0;
    const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
    const int step = j >> 1, half = j & 1;
#pragma unroll 1
    for (int ci = 0; ci < nxc; ++ci) {
        const int fmt = p.xf[ci];
        const int sb = s_pos(fmt, j * 8, p.H);
        const float sc = __int_as_float((127 + sh.xn[c] - sb) << 23);
        float sum = 0.f;
        uint8_t* dst = xh + (ci * p.T + c) * p.x_stride + step * 32 + half * 4;
#pragma unroll
        for (int tp = 0; tp < 4; ++tp) {
            const __half2 h = __floats2half2_rn(__uint_as_float(wv[tp] << 16) * sc,
                                                __uint_as_float(wv[tp] & 0xffff0000u) * sc);
            if (in) *reinterpret_cast<__half2*>(dst + tp * 8) = h;
            sum += __low2float(h) + __high2float(h);
        }
        sum *= __int_as_float((127 + sb) << 23);
        sum += __shfl_xor_sync(0xffffffffu, sum, 1);
        sum += __shfl_xor_sync(0xffffffffu, sum, 2);
        if (in && (lane & 3) == 0) sx[(ci * p.T + c) * sxs + (j >> 2)] = sum;
    }
}

// Chained input (the next layer of a stack): x = bf16(y / r), r = sqrt of the
// mean of y^2 per column, bit for bit what moe_rms_norm_bf16 gives: the sum
// of squares in its order (threads 0..255, element i on thread i mod 256,
// fp64 fma, then the two warp trees) and the nearest-even bf16 of the fp64
// quotient y / r.
__device__ void chain_rms(const MoeParams& p, Shared& sh, int sid, int nthr) {
    const int lane = sid & 31;
    if (sid < 256) {
        for (int c = 0; c < p.T; ++c) {
            const float* yc = p.xc + (long long)c * p.H;
            double ss = 0.0;
            for (int i = sid; i < p.H; i += 256) {
                const double v = (double)__ldg(yc + i);
                ss = fma(v, v, ss);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
            if (lane == 0) sh.rms_part[c][sid >> 5] = ss;
        }
    }
    asm volatile("bar.sync 1, %0;" ::"r"(nthr) : "memory");
    if (sid < 32) {
        for (int c = 0; c < p.T; ++c) {
            double t = lane < 8 ? sh.rms_part[c][lane] : 0.0;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
            if (lane == 0) {
                const double r = sqrt(t / (double)p.H);
                sh.rms_r[c] = r;
                sh.rms_ri[c] = 1.0 / r;
            }
        }
    }
    asm volatile("bar.sync 1, %0;" ::"r"(nthr) : "memory");
}

// bf16 bits of y / r.  The product y * (1/r) is within 3 fp64 ulps of the
// rounded quotient; unless it lies within half an fp32 ulp (plus that margin)
// of a bf16 rounding tie, or outside the normal bf16 range, its bf16 through
// fp32 (two nearest-even steps) equals the quotient's.  Otherwise divide.
// The division is out of line: it is rare, and inlined at every use it would
// be most of the kernel's code.
__device__ __noinline__ uint32_t chain_bf16_div(float y, double r) { return f64_to_bf16_rne((double)y / r); }

__device__ __forceinline__ uint32_t chain_bf16(float y, double r, double ri) {
    const double q = (double)y * ri;
    const unsigned long long b = (unsigned long long)__double_as_longlong(q);
    const int e = (int)((b >> 52) & 0x7FF);
    const long long d = (long long)(b & ((1ull << 45) - 1ull)) - (1ll << 44);
    constexpr long long WIN = (1ll << 28) + 8;
    if (e < 1023 - 126 || e == 0x7FF || (d < WIN && d > -WIN)) return chain_bf16_div(y, r);
    return __bfloat16_as_ushort(__float2bfloat16_rn(__double2float_rn(q)));
}

// Item i (8 consecutive values of a column) of the chained input as bf16
// bits (inlined only in the chained branch of load_round).
__device__ __forceinline__ uint4 load_item_chained(const MoeParams& p, const Shared& sh, int i, int per_col) {
    const int c = i / per_col;
    const float4 a = __ldg(reinterpret_cast<const float4*>(p.xc) + 2 * i);
    const float4 b = __ldg(reinterpret_cast<const float4*>(p.xc) + 2 * i + 1);
    const double r = sh.rms_r[c], ri = sh.rms_ri[c];
    return make_uint4(chain_bf16(a.x, r, ri) | (chain_bf16(a.y, r, ri) << 16),
                      chain_bf16(a.z, r, ri) | (chain_bf16(a.w, r, ri) << 16),
                      chain_bf16(b.x, r, ri) | (chain_bf16(b.y, r, ri) << 16),
                      chain_bf16(b.z, r, ri) | (chain_bf16(b.w, r, ri) << 16));
}

// The items r0 + sid + k * nthr (k < XR) of x as bf16 bits, zero past the
// end.  The test of the chained input is outside the loads: the plain path is
// XR loads in flight and nothing else.
__device__ __forceinline__ void load_round(const MoeParams& p, const Shared& sh, int r0, int sid, int nthr, int nitems,
                                           int per_col, uint4 v[XR]) {
    if (!p.xc) {
#pragma unroll
        for (int k = 0; k < XR; ++k) {
            const int i = r0 + sid + k * nthr;
            v[k] = i < nitems ? __ldg(reinterpret_cast<const uint4*>(p.x) + i) : make_uint4(0u, 0u, 0u, 0u);
        }
    } else {
#pragma unroll
        for (int k = 0; k < XR; ++k) {
            const int i = r0 + sid + k * nthr;
            v[k] = i < nitems ? load_item_chained(p, sh, i, per_col) : make_uint4(0u, 0u, 0u, 0u);
        }
    }
}

__device__ void stage_x(const MoeParams& p, Shared& sh, uint8_t* xh, int sid, int nthr) {
    const int lane = sid & 31;
    const int per_col = p.H / 8;
    const uint32_t cdiv = 0xffffffffu / (uint32_t)per_col + 1u;
    const int nitems = p.T * per_col;
    if (p.xc) chain_rms(p, sh, sid, nthr);
    const int nxc = p.nxc;
    float* sx = (float*)(xh + nxc * p.T * p.x_stride);
    const int sxs = moe_sxs(p.H);
    const bool one_round = nitems <= XR * nthr;   // then pass 2 reuses the loaded items
    uint4 v[XR];
    // pass 1: max |x| per column
    for (int r0 = 0; r0 < nitems; r0 += XR * nthr) {
        load_round(p, sh, r0, sid, nthr, nitems, per_col, v);
#pragma unroll
        for (int k = 0; k < XR; ++k) {
            const int i0 = r0 + k * nthr + sid - lane;
            if (i0 < nitems) x_max(sh, v[k], i0, lane, nitems, cdiv);
        }
    }
    asm volatile("bar.sync 1, %0;" ::"r"(nthr) : "memory");
    if (sid < p.T) {
        const uint32_t mm = sh.xmax[sid];
        const int n = mm ? 13 - ((int)((mm >> 23) & 255u) - 127) : 0;
        sh.xn[sid] = max(-100, min(100, n));
    }
    asm volatile("bar.sync 1, %0;" ::"r"(nthr) : "memory");
    // pass 2: scale, round to fp16, write fragments and block sums.  One copy
    // of the code (it runs once per launch, its instructions not yet cached):
    // a rolled loop over the round's items.  With one round the items are
    // still in registers from pass 1 (picked with static indices); else they
    // are loaded again.
    for (int r0 = 0; r0 < nitems; r0 += XR * nthr) {
        if (!one_round) load_round(p, sh, r0, sid, nthr, nitems, per_col, v);
#pragma unroll 1
        for (int k = 0; k < XR; ++k) {
            const int i0 = r0 + k * nthr + sid - lane;   // warp-uniform
            if (i0 >= nitems) break;
            uint4 cur = v[0];
#pragma unroll
            for (int j = 1; j < XR; ++j)
                if (k == j) cur = v[j];
            x_put(p, sh, xh, sx, sxs, nxc, cur, i0, lane, nitems, per_col, cdiv);
        }
    }
}

// ---------------------------------------------------------------- kernel ---

template <int QC, bool OTHER>
__global__ void __launch_bounds__(NTHREADS, 1) moe_decode_kernel(MoeParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* ring = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t* xh = ring + p.ns * MOE_STAGE_BYTES;
    uint8_t* red = xh + p.xh_bytes;
    Shared& sh = *(Shared*)(red + p.nred * 2 * moe_red_bytes(QC));
    const int w = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    grid_dep_launch();   // the next kernel may launch (it waits for this one before its loads)
    if (threadIdx.x == 0) {
        for (int s = 0; s < p.ns; ++s) {
            mbar_init(&sh.full[s], 1);
            mbar_init(&sh.empty[s], NCW);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sh.hfull[i], 1);
            mbar_init(&sh.hfree[i], NCW);
        }
        for (int i = 0; i < p.nred; ++i) {
            mbar_init(&sh.rfull[i], NCW);
            mbar_init(&sh.rempty[i], 1);
        }
        sh.abort_flag = 0;
        sh.consumed = 0;
        sh.bar_ok = 0;
        for (int c = 0; c < MOE_MAXT; ++c) sh.xmax[c] = 0u;
        fence_barrier_init();
    }
    __syncthreads();
    // The shared expert's first gate/up unit (this CTA's first) depends on
    // nothing the previous kernel writes: stream as many of its stages as the
    // ring holds now (the consumers free none before the routing is known).
    ProdRing q;
    int last_a = -1, pre = 0;
    if (w == WARP_PRODUCER && lane == 0 && p.has_shared && (int)blockIdx.x < p.I / 32) {
        const int k1 = min(a_stages(p.H), p.ns);
        if (issue_a(p, sh, ring, q, 0, -1, (int)blockIdx.x, 0, k1, policy_evict_first(), last_a)) {
            pre = k1;
        } else {
            set_error(p.ctrl, MOE_ERR_TIMEOUT);
            sh.abort_flag = 1;
        }
    }
    // everything below may read what the previous kernel wrote (routing, x,
    // the workspace)
    grid_dep_wait();
    if (w == WARP_PRODUCER) {
        const Routing rt = load_routing(p);
        build_slots(p, sh.st, rt);
        asm volatile("bar.arrive 2, %0;" ::"n"(NTHREADS) : "memory");
        if (lane == 0 && !sh.abort_flag) producer(p, sh, ring, xh, q, pre, last_a);
    } else {
        const int sid = w < WARP_PRODUCER ? threadIdx.x : threadIdx.x - 32;
        stage_x(p, sh, xh, sid, NSTAGE_THREADS);
        asm volatile("bar.sync 2, %0;" ::"n"(NTHREADS) : "memory");
        if (w < NCW) consumer<QC, OTHER>(p, sh, ring, xh, red);
        else epilogue_warp<QC>(p, sh, red, w - WARP_EPI0);
    }
    __syncthreads();
    // every partial of this CTA is stored; wait for all CTAs' (the one grid barrier)
    if (threadIdx.x == 0) {
        bool ok = !sh.abort_flag;
        if (ok) {
            __threadfence();
            ok = grid_barrier(reinterpret_cast<unsigned long long*>(p.ctrl + MOE_CTRL_BAR), p.wait_limit,
                              p.fault == 1 ? 1 : 0);
            if (!ok) set_error(p.ctrl, MOE_ERR_TIMEOUT);
        }
        sh.bar_ok = ok ? 1 : 0;
    }
    __syncthreads();
    if (!sh.bar_ok) return;
    const SlotTable& S = sh.st;
    // CTA 0 returns the per-launch counters to zero (every CTA is past its last use)
    if (blockIdx.x == 0) {
        for (int i = threadIdx.x; i < S.nslots; i += NTHREADS) p.ctrl[MOE_CTRL_SLOT_DONE + i] = 0u;
        if (threadIdx.x == 0) p.ctrl[MOE_CTRL_QUEUE] = 0u;
    }
    // combine: y[c] = sum_j w[c][j] * partial[slot(c, j)] + partial[shared], in
    // the fixed order j = 0 .. k-1 then the shared expert (column c does not
    // depend on T); this CTA owns elements [n b / G, n (b+1) / G)
    const long long n = (long long)p.T * p.H;
    const int i0 = (int)(n * blockIdx.x / gridDim.x), i1 = (int)(n * (blockIdx.x + 1) / gridDim.x);
    for (int i = i0 + threadIdx.x; i < i1; i += NTHREADS) {
        const int c = i / p.H, r = i - c * p.H;
        float v[MOE_MAXK];
#pragma unroll
        for (int j = 0; j < MOE_MAXK; ++j) {
            const int s2 = j < p.k ? S.tslot[c][j] : -1;
            v[j] = s2 >= 0 ? __ldcg(p.dpart + ((long long)s2 * p.T + S.tpos[c][j]) * p.H + r) : 0.f;
        }
        const float vs = p.has_shared ? __ldcg(p.dpart + (long long)c * p.H + r) : 0.f;
        float acc = 0.f;
#pragma unroll
        for (int j = 0; j < MOE_MAXK; ++j)
            if (j < p.k && S.tslot[c][j] >= 0) acc = fmaf(S.w[c][j], v[j], acc);
        if (p.has_shared) acc += vs;
        p.y[i] = acc;
    }
}

// Shared-memory bytes of a launch (plus 1 KB alignment slack).
size_t moe_decode_smem_bytes(int ns, int nred, int xh_bytes, int qc) {
    return 1024 + (size_t)ns * MOE_STAGE_BYTES + xh_bytes + (size_t)nred * 2 * moe_red_bytes(qc) + sizeof(Shared);
}

cudaError_t moe_decode_launch(const MoeParams& p, int grid, cudaStream_t stream) {
    const int qc = moe_qclass(p.T);
    const size_t smem = moe_decode_smem_bytes(p.ns, p.nred, p.xh_bytes, qc);
    void (*kerns[2][3])(MoeParams) = {{moe_decode_kernel<1, false>, moe_decode_kernel<2, false>, moe_decode_kernel<3, false>},
                                       {moe_decode_kernel<1, true>, moe_decode_kernel<2, true>, moe_decode_kernel<3, true>}};
    const int ot = p.other ? 1 : 0;
    auto kern = kerns[ot][qc - 1];
    // the dynamic shared-memory limit, once per device and kernel
    static SmemLimit limit[2][3];
    cudaError_t err = limit[ot][qc - 1].ensure((const void*)kern, (int)smem);
    if (err != cudaSuccess) return err;
    // cooperative: every CTA is resident at once (the final grid barrier needs it)
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(NTHREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute at[2];
    at[0].id = cudaLaunchAttributeCooperative;
    at[0].val.cooperative = 1;
    // programmatic dependent of the kernel before it (the router): the CTAs
    // start, set up and stream the shared expert while it finishes, and wait
    // for it before any load of its outputs
    at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kern, p);
}

long long moe_default_wait_limit() { return DEFAULT_WAIT; }

}  // namespace rfx
