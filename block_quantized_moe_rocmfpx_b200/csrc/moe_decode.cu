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
//  - One persistent kernel, one CTA per SM, three phases: (A) gate/up
//    row-groups -> SwiGLU -> h of every slot, (B) down row-groups -> per-slot
//    partial outputs, (C) fixed-order weighted combine -> y.  Each CTA owns a
//    contiguous, cost-balanced range of 16-row groups in A and in B
//    (slot-major, so a CTA's row-groups share an x column set or an h
//    buffer).  The phases meet at two grid barriers (one release-add and one
//    acquire poll per CTA each); the weight stream does not stop at the
//    first one: the producer runs straight on into the down weights, only
//    the copy of h waits for it.
//  - Per CTA: one lane of the producer warp streams spans of 8 chunks HBM ->
//    shared memory with 1-D bulk copies (TMA, evict-first L2 policy) into a
//    ring of stages, each with a record of what it holds (8 gate + 8 up
//    chunks, or two down row-groups of up to 8 chunks).  8 consumer warps
//    take one chunk of each half of every stage, decode it in registers (one
//    AND per A register, see rfx_tile.cuh) and run mma.sync m16n8k16 in fp16:
//    x normalised per column by a power of two for gate/up, an exact hi/lo
//    fp16 split of h for down.  2 epilogue warps sum the 8 warps' partials of
//    each row-group in a fixed order and run SwiGLU (A) or store the partial
//    (B), then run the combine (C).
//  - Every wait is bounded; a timeout sets a workspace error flag and the CTA
//    drains its in-flight copies and exits.
#include <cuda_runtime.h>

#include "launch_util.h"
#include "moe_decode.h"
#include "rfx_tile.cuh"

namespace rfx {

constexpr int NCW = 8;                       // consumer warps 0..7
constexpr int WARP_PRODUCER = NCW;           // weight bulk copies (one lane)
constexpr int WARP_HLOAD = NCW + 1;          // first grid barrier, then h bulk copies (one lane)
constexpr int NEPI = 2;                      // epilogue warps: reductions, SwiGLU / partial stores, combine
constexpr int WARP_EPILOGUE0 = NCW + 2;
constexpr int NTHREADS = (NCW + 2 + NEPI) * 32;
constexpr int NRED_MAX = MOE_MAX_RED;        // reduction buffers: unit r -> buffer r % nred,
                                             // epilogue warp r % NEPI
constexpr long long WAIT_LIMIT = 4000000000LL;

struct __align__(16) SlotTable {
    float w[MOE_MAXT][MOE_MAXK];              // routing weights
    signed char tslot[MOE_MAXT][MOE_MAXK];    // slot of (column, j), -1 if invalid
    signed char tpos[MOE_MAXT][MOE_MAXK];     // position of the column among the slot's columns
    int nslots;
    int expert[MOE_MAXS];                     // -1: shared expert
    int ncols[MOE_MAXS];
    unsigned colmask[MOE_MAXS];               // columns routed to the slot (bit c)
    signed char cols[MOE_MAXS][MOE_MAXT];
    unsigned mask[32];                        // experts in use (bit per expert)
    int prefix[32];
    int idx[MOE_MAXT * MOE_MAXK];
};

// A reduction unit: a row-group's partials from the 8 consumer warps, or a
// marker (end of the gate/up phase, end of work).
enum : int { UNIT_A = 0, UNIT_B = 1, UNIT_A_END = 2, UNIT_END = 3 };
struct RedInfo {
    int kind, slot, ncols, rg;
};

// What a ring stage holds, written by the producer with the stage.
enum : short { REC_FIRST = 1, REC_LAST = 2, REC_HNEW = 4, REC_HDONE = 8, REC_END = 16 };
struct __align__(16) StageRec {
    short kind;    // 0: gate + up span, 1: down span(s)
    short slot;
    short rg;      // row-group of the matrix (rows 16*rg ..); down: first of n
    short c0;      // first chunk of the span
    short n;       // down: row-groups in the stage (one per half)
    short flags;   // REC_*: first / last span of the row-group(s); first / last stage of a slot's h
    short hseq;    // down: index of the slot in this CTA's range (h buffer hseq & 1)
    short pad;
};

struct Shared {
    uint64_t full[MOE_MAX_STAGES];
    uint64_t empty[MOE_MAX_STAGES];
    uint64_t hfull[2], hfree[2];
    uint64_t rfull[NRED_MAX], rempty[NRED_MAX];
    uint64_t adone;          // both epilogue warps are past the gate/up phase
    uint64_t xload;          // bulk copy of x into the (not yet used) reduction buffers
    RedInfo rinfo[NRED_MAX];
    StageRec rec[MOE_MAX_STAGES];
    volatile int abort_flag;
    volatile int consumed;   // stages released by all consumer warps (for the abort drain)
    int bar_ok;              // second grid barrier passed (epilogue warps)
    int ub0, ub1;            // this CTA's down row-groups
    unsigned xmax[MOE_MAXT]; // max |x| per column (fp32 bits)
    int xn[MOE_MAXT];        // x is staged as x * 2^xn[c] (then 2^-s_b per tile position)
    SlotTable st;
};

__device__ __forceinline__ void set_error(uint32_t* ctrl, uint32_t bits) { atomicOr(ctrl + MOE_CTRL_ERR, bits); }

// The routing of the T columns, loaded by the producer warp's lanes before
// anything else (lane L holds entries L and L + 32 of idx / w).
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

// Union of routed experts over the T columns for T * k <= 32 (one warp, one
// entry per lane, no loops): slot 0 is the shared expert (if any), then the
// distinct valid experts in order of first appearance (column-major).
__device__ void build_slots_small(const MoeParams& p, SlotTable& S, const Routing& rt) {
    const int lane = threadIdx.x & 31;
    const unsigned lt = (1u << lane) - 1u;
    const int n = p.T * p.k;
    const int base = p.has_shared ? 1 : 0;
    const int c = lane / p.k, j = lane - c * p.k;
    const int e = rt.e0;
    const bool in = lane < n;
    bool v = in && e >= 0 && e < p.E;
    if (in && !v) set_error(p.ctrl, MOE_ERR_EXPERT);
    // an expert repeated within a column counts once (the later entries are flagged)
    const unsigned same = __match_any_sync(0xffffffffu, v ? e : -1 - lane);
    const unsigned col_lanes = ((1u << p.k) - 1u) << (c * p.k);
    if (v && (same & lt & col_lanes)) {
        v = false;
        set_error(p.ctrl, MOE_ERR_DUP);
    }
    const unsigned grp = __match_any_sync(0xffffffffu, v ? e : -1 - lane);   // valid entries of the same expert
    const bool first = v && !(grp & lt);
    const unsigned firsts = __ballot_sync(0xffffffffu, first);
    int slot = base + __popc(firsts & lt);
    slot = __shfl_sync(0xffffffffu, slot, __ffs(grp) - 1);
    const int pos = __popc(grp & lt);            // earlier columns of this expert
    if (in) {
        S.w[c][j] = rt.w0;
        S.tslot[c][j] = v ? (signed char)slot : (signed char)-1;
        S.tpos[c][j] = (signed char)pos;
    }
    if (v) S.cols[slot][pos] = (signed char)c;
    if (first) {
        S.expert[slot] = e;
        S.ncols[slot] = __popc(grp);
    }
    if (lane == 0) {
        S.nslots = base + __popc(firsts);
        if (p.has_shared) {
            S.expert[0] = -1;
            S.ncols[0] = p.T;
            for (int cc = 0; cc < p.T; ++cc) S.cols[0][cc] = (signed char)cc;
        }
    }
    __syncwarp();
}

// Union of routed experts over the T columns (one warp), any T * k <= 64:
// slot 0 is the shared expert (if any), then the distinct valid experts in
// ascending order.
__device__ void build_slots(const MoeParams& p, SlotTable& S, const Routing& rt) {
    const int lane = threadIdx.x & 31;
    const int n = p.T * p.k;
    const int base = p.has_shared ? 1 : 0;
    S.mask[lane] = 0u;
    for (int s = lane; s < MOE_MAXS; s += 32) S.colmask[s] = 0u;
    if (lane < n) { S.idx[lane] = rt.e0; S.w[lane / p.k][lane % p.k] = rt.w0; }
    if (lane + 32 < n) { S.idx[lane + 32] = rt.e1; S.w[(lane + 32) / p.k][(lane + 32) % p.k] = rt.w1; }
    __syncwarp();
    bool ok[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        const int i = lane + 32 * h;
        ok[h] = false;
        if (i >= n) continue;
        const int c = i / p.k, j = i - (i / p.k) * p.k;
        const int e = S.idx[i];
        bool v = e >= 0 && e < p.E;
        if (!v) set_error(p.ctrl, MOE_ERR_EXPERT);
        for (int jj = 0; jj < j && v; ++jj)
            if (S.idx[c * p.k + jj] == e) { v = false; set_error(p.ctrl, MOE_ERR_DUP); }
        ok[h] = v;
        S.tslot[c][j] = -1;
        if (v) atomicOr(&S.mask[e >> 5], 1u << (e & 31));
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
    int slot_of[2] = {-1, -1};
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        if (!ok[h]) continue;
        const int i = lane + 32 * h;
        const int e = S.idx[i];
        const int s = base + S.prefix[e >> 5] + __popc(S.mask[e >> 5] & ((1u << (e & 31)) - 1u));
        slot_of[h] = s;
        S.expert[s] = e;
        atomicOr(&S.colmask[s], 1u << (i / p.k));
    }
    __syncwarp();
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        if (slot_of[h] < 0) continue;
        const int i = lane + 32 * h;
        const int c = i / p.k, j = i - c * p.k, s = slot_of[h];
        const unsigned cm = S.colmask[s];
        const int pos = __popc(cm & ((1u << c) - 1u));   // columns ascend within a slot
        S.cols[s][pos] = (signed char)c;
        S.tslot[c][j] = (signed char)s;
        S.tpos[c][j] = (signed char)pos;
        if (pos == 0) S.ncols[s] = __popc(cm);
    }
    if (p.has_shared && lane == 0) {
        S.expert[0] = -1;
        S.ncols[0] = p.T;
        S.colmask[0] = (1u << p.T) - 1u;
        for (int c = 0; c < p.T; ++c) S.cols[0][c] = (signed char)c;
    }
    __syncwarp();
}

// Packed stream of the gate/up (phase 0) or down (phase 1) matrices of a slot.
struct MatRef {
    const uint8_t* a;
    const uint8_t* b;
    int fmt;
};

__device__ __forceinline__ MatRef slot_mats(const MoeParams& p, int e, int ph) {
    if (ph == 0) {
        if (e < 0) return {p.shg, p.shu, p.fsA};
        return {p.gate + (long long)e * p.sg, p.up + (long long)e * p.su, p.fA};
    }
    if (e < 0) return {p.shd, nullptr, p.fsB};
    return {p.down + (long long)e * p.sd, nullptr, p.fB};
}

// ------------------------------------------------------------ partition ---
//
// Down row-groups ("units") are numbered slot-major: u = slot * nrg + rg.
// They are split statically (each CTA copies the h of only the one or two
// slots of its range): CTA b owns the units whose starting cost lies in
// [total * b / G, total * (b+1) / G).  All units have the same tiles; their
// cost depends on the format only (measured decode + mma cycles per tile of
// this implementation, relative units), so there are two unit costs: the
// shared expert's (slot 0, if any) and the routed experts'.
__device__ __forceinline__ int down_cost(int fmt) { return fmt == 2 ? 70 : (fmt == 3 ? 81 : 94); }

__device__ void down_units(const MoeParams& p, int nslots, int& u0, int& u1) {
    const int nrg = p.H / 16;
    const int ns = p.has_shared ? 1 : 0, nr = nslots - ns;
    const int cs = down_cost(p.fsB), cr = down_cost(p.fB);
    const long long shared_total = (long long)ns * nrg * cs;
    const long long total = shared_total + (long long)nr * nrg * cr;
    auto unit_at = [&](long long target) -> int {   // first unit whose starting cost is >= target
        if (target < shared_total) return (int)((target + cs - 1) / cs);
        const long long k = (target - shared_total + cr - 1) / cr;
        return ns * nrg + (int)min(k, (long long)nr * nrg);
    };
    u0 = unit_at(total * blockIdx.x / gridDim.x);
    u1 = unit_at(total * (blockIdx.x + 1) / gridDim.x);
}

// ------------------------------------------------------------- producer ---
//
// Gate/up: per row-group, one stage per span of up to 8 chunks (one bulk copy
// of the span per matrix, gate in the first half of the stage, up in the
// second).  Down: when a row-group fits one half (at most 8 chunks), a stage
// holds two consecutive row-groups of a slot, else spans of 8 chunks.  The
// stage record is written before the arrive that publishes the stage, so a
// consumer reads it after its acquire on `full`.

struct ProdRing {
    int stage = 0, n = 0;
    uint32_t phase = 1;   // producer: parity to wait for on empty[stage] (fresh barriers pass)
};

__device__ __forceinline__ bool claim(const MoeParams& p, Shared& sh, ProdRing& rg) {
    return mbar_wait(&sh.empty[rg.stage], rg.phase, WAIT_LIMIT);
}

__device__ __forceinline__ void advance(const MoeParams& p, ProdRing& rg) {
    ++rg.n;
    if (++rg.stage == p.ns) { rg.stage = 0; rg.phase ^= 1u; }
}

// Gate/up row-groups are handed out dynamically (a global counter), one at a
// time, so CTAs that run faster take more; they are numbered slot-major, the
// shared expert (the largest units) first, and the next grab is always in
// flight while the current row-group streams.  Down row-groups come from the
// CTA's static range.
__device__ void producer(const MoeParams& p, Shared& sh, uint8_t* ring) {
    const SlotTable& S = sh.st;
    const uint64_t pol_w = policy_evict_first();
    ProdRing q;
    bool ok = true;
    // ---- gate/up
    {
        const int nrg = p.I / 16, nch = rfx_num_chunks(p.H);
        const int nunits = S.nslots * nrg;
        int next = (int)atomicAdd(p.ctrl + MOE_CTRL_TASK_A, 1u);
        while (ok) {
            const int u = next;
            if (u >= nunits) break;
            next = (int)atomicAdd(p.ctrl + MOE_CTRL_TASK_A, 1u);
            const int slot = u / nrg, rg = u - slot * nrg;
            const MatRef m = slot_mats(p, S.expert[slot], 0);
            const long long rgb = rfx_rowgroup_bytes(m.fmt, p.H);
            const int fullb = (int)rfx_chunk_bytes(m.fmt, 8);
            const uint32_t lastb = (uint32_t)rfx_chunk_bytes(m.fmt, rfx_chunk_tiles(p.H, nch - 1));
            for (int c0 = 0; c0 < nch; c0 += MOE_CHUNKS_PER_STAGE) {
                const int c1 = min(nch, c0 + MOE_CHUNKS_PER_STAGE);
                const uint32_t bytes = (uint32_t)((c1 - 1 - c0) * fullb) + (c1 == nch ? lastb : (uint32_t)fullb);
                if (!claim(p, sh, q)) { ok = false; break; }
                StageRec r{};
                r.kind = 0;
                r.slot = (short)slot;
                r.rg = (short)rg;
                r.c0 = (short)c0;
                r.n = 1;
                r.flags = (short)((c0 == 0 ? REC_FIRST : 0) | (c1 == nch ? REC_LAST : 0));
                sh.rec[q.stage] = r;
                uint8_t* dst = ring + q.stage * MOE_STAGE_BYTES;
                const long long off = (long long)rg * rgb + (long long)c0 * fullb;
                mbar_arrive_expect_tx(&sh.full[q.stage], 2 * bytes);
                bulk_g2s(dst, m.a + off, bytes, &sh.full[q.stage], pol_w);
                bulk_g2s(dst + MOE_HALF_BYTES, m.b + off, bytes, &sh.full[q.stage], pol_w);
                advance(p, q);
            }
        }
    }
    // ---- down (needs nothing of the gate/up phase: no barrier here)
    {
        const int nrg = p.H / 16, nch = rfx_num_chunks(p.I);
        int hseq = -1, prev_slot = -1;
        for (int u = sh.ub0; u < sh.ub1 && ok;) {
            const int slot = u / nrg, rg = u - slot * nrg;
            if (slot != prev_slot) { ++hseq; prev_slot = slot; }
            const MatRef m = slot_mats(p, S.expert[slot], 1);
            const long long rgb = rfx_rowgroup_bytes(m.fmt, p.I);
            const int fullb = (int)rfx_chunk_bytes(m.fmt, 8);
            const uint32_t lastb = (uint32_t)rfx_chunk_bytes(m.fmt, rfx_chunk_tiles(p.I, nch - 1));
            const bool hnew = (u == sh.ub0) || rg == 0;
            if (nch <= MOE_CHUNKS_PER_STAGE) {
                // one stage holds two consecutive row-groups of the slot (one per half)
                const int pair = (u + 1 < sh.ub1 && (u + 1) / nrg == slot) ? 2 : 1;
                const int ul = u + pair - 1;
                const bool hdone = (ul + 1 == sh.ub1) || ((ul + 1) / nrg != slot);
                if (!claim(p, sh, q)) { ok = false; break; }
                StageRec r{};
                r.kind = 1;
                r.slot = (short)slot;
                r.rg = (short)rg;
                r.c0 = 0;
                r.n = (short)pair;
                r.flags = (short)(REC_FIRST | REC_LAST | (hnew ? REC_HNEW : 0) | (hdone ? REC_HDONE : 0));
                r.hseq = (short)hseq;
                sh.rec[q.stage] = r;
                uint8_t* dst = ring + q.stage * MOE_STAGE_BYTES;
                mbar_arrive_expect_tx(&sh.full[q.stage], (uint32_t)(pair * rgb));
                for (int i = 0; i < pair; ++i)
                    bulk_g2s(dst + i * MOE_HALF_BYTES, m.a + (long long)(rg + i) * rgb, (uint32_t)rgb, &sh.full[q.stage],
                             pol_w);
                advance(p, q);
                u += pair;
            } else {
                const bool hdone = (u + 1 == sh.ub1) || ((u + 1) / nrg != slot);
                for (int c0 = 0; c0 < nch; c0 += MOE_CHUNKS_PER_STAGE) {
                    const int c1 = min(nch, c0 + MOE_CHUNKS_PER_STAGE);
                    const uint32_t bytes = (uint32_t)((c1 - 1 - c0) * fullb) + (c1 == nch ? lastb : (uint32_t)fullb);
                    if (!claim(p, sh, q)) { ok = false; break; }
                    StageRec r{};
                    r.kind = 1;
                    r.slot = (short)slot;
                    r.rg = (short)rg;
                    r.c0 = (short)c0;
                    r.n = 1;
                    r.flags = (short)((c0 == 0 ? REC_FIRST : 0) | (c1 == nch ? REC_LAST : 0) |
                                      (c0 == 0 && hnew ? REC_HNEW : 0) | (c1 == nch && hdone ? REC_HDONE : 0));
                    r.hseq = (short)hseq;
                    sh.rec[q.stage] = r;
                    uint8_t* dst = ring + q.stage * MOE_STAGE_BYTES;
                    mbar_arrive_expect_tx(&sh.full[q.stage], bytes);
                    bulk_g2s(dst, m.a + (long long)rg * rgb + (long long)c0 * fullb, bytes, &sh.full[q.stage], pol_w);
                    advance(p, q);
                }
                ++u;
            }
        }
    }
    // end-of-work record: a stage with no copy
    if (ok) {
        if (claim(p, sh, q)) {
            StageRec r{};
            r.kind = -1;
            r.flags = REC_END;
            sh.rec[q.stage] = r;
            mbar_arrive(&sh.full[q.stage]);
        } else {
            ok = false;
        }
    }
    if (!ok) {
        set_error(p.ctrl, MOE_ERR_TIMEOUT);
        sh.abort_flag = 1;
        // drain: wait (bounded) until every issued copy has landed
        for (int i = sh.consumed; i < q.n; ++i) (void)mbar_wait(&sh.full[i % p.ns], (i / p.ns) & 1, WAIT_LIMIT);
    }
}

// ----------------------------------------------------------- grid barrier ---
//
// One thread per CTA: a release add on a 64-bit counter that only grows, then
// an acquire poll until every CTA of this launch has added.  The target is the
// next multiple of the grid size above the value this CTA saw, so the counter
// needs no reset between calls (a timed-out call leaves it unaligned: the
// workspace must then be re-initialised).  Returns false on timeout.
__device__ bool grid_barrier(unsigned long long* ctr) {
    const unsigned long long G = gridDim.x;
    const unsigned long long old = atom_add_release_gpu_u64(ctr, 1ull);
    const unsigned long long target = (old / G + 1) * G;
    const long long t0 = clock64();
    unsigned nap = 32;
    while (ld_acquire_gpu_u64(ctr) < target) {
        if (clock64() - t0 > WAIT_LIMIT) return false;
        __nanosleep(nap);
        nap = min(nap * 2u, 256u);
    }
    return true;
}

// The h lane: once every CTA has written its h (first grid barrier), for
// each slot of the CTA's down range, in order, bulk-copy the slot's h and
// block sums into buffer (slot index & 1) once the consumers released it.
// CTA 0 also resets the gate/up task counter (every CTA has taken its last
// gate/up row-group before it arrives).
__device__ void h_loader(const MoeParams& p, Shared& sh, uint8_t* xh, int hbytes_max, int sstr) {
    const SlotTable& S = sh.st;
    bool ok = mbar_wait(&sh.adone, 0, WAIT_LIMIT) &&
              grid_barrier(reinterpret_cast<unsigned long long*>(p.ctrl + MOE_CTRL_BAR_H));
    if (ok && blockIdx.x == 0) p.ctrl[MOE_CTRL_TASK_A] = 0u;
    int n = 0;
    if (ok && sh.ub0 < sh.ub1) {
        fence_proxy_async_global();   // generic-proxy writes of h (other CTAs) -> bulk-copy reads
        const uint64_t pol_h = policy_evict_last();
        const int nrg = p.H / 16;
        const int s0 = sh.ub0 / nrg, s1 = (sh.ub1 - 1) / nrg;
        for (int slot = s0; slot <= s1; ++slot, ++n) {
            const int buf = n & 1;
            if (!mbar_wait(&sh.hfree[buf], ((n >> 1) + 1) & 1, WAIT_LIMIT)) { ok = false; break; }
            const uint32_t hb = 4u * (uint32_t)S.ncols[slot] * (uint32_t)(p.I + sstr);
            mbar_arrive_expect_tx(&sh.hfull[buf], hb);
            bulk_g2s(xh + buf * hbytes_max, p.hbuf + (long long)slot * (2LL * p.T * (p.I + sstr)), hb,
                     &sh.hfull[buf], pol_h);
        }
    }
    if (!ok) {
        set_error(p.ctrl, MOE_ERR_TIMEOUT);
        sh.abort_flag = 1;
        for (int b = 0; b < 2 && b < n; ++b)
            (void)mbar_wait(&sh.hfull[(n - 1 - b) & 1], ((n - 1 - b) >> 1) & 1, WAIT_LIMIT);
    }
}

// ------------------------------------------------------------- epilogues ---

// A reduction buffer holds the 8 consumer warps' partials of one unit as
// [warp][half][lane][4 floats]: every 128-bit access of a warp covers 512
// contiguous bytes (no bank conflicts).  Sums them in warp order.
__device__ __forceinline__ void red_sum(const float* rb0, int lane, float lo[4], float hi[4]) {
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
#pragma unroll
    for (int w = 0; w < NCW; ++w) {
        const float4 x = ldsf4((const uint8_t*)(rb0 + ((w * 2 + 0) * 32 + lane) * 4));
        const float4 y = ldsf4((const uint8_t*)(rb0 + ((w * 2 + 1) * 32 + lane) * 4));
        a.x += x.x; a.y += x.y; a.z += x.z; a.w += x.w;
        b.x += y.x; b.y += y.y; b.z += y.z; b.w += y.w;
    }
    lo[0] = a.x; lo[1] = a.y; lo[2] = a.z; lo[3] = a.w;
    hi[0] = b.x; hi[1] = b.y; hi[2] = b.z; hi[3] = b.w;
}

// SwiGLU of one row-group: undo the per-column x scaling, h = silu(g) * u,
// store h as an fp16 hi/lo pair in the fragment order of the down projection's
// B operand ([step][v][t'][4], v = 2*col + {0 hi, 1 lo}) and the row-group's
// sum of (hi + lo) per column (half of a 32-wide down block).
__device__ void epilogue_a(const MoeParams& p, const Shared& sh, const float* rb0, int slot, int ncols, int rg,
                           int lane, int sstr) {
    const int g = lane >> 2, t = lane & 3;
    uint16_t* hs = p.hbuf + (long long)slot * (2LL * p.T * (p.I + sstr));
    float* hsum = (float*)(hs + 2LL * ncols * p.I);
    float G[4], U[4];
    red_sum(rb0, lane, G, U);
    uint32_t bad = 0;
    const int step = rg;
    float part[2] = {0.f, 0.f};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int col = 2 * t + (i & 1);
        const int rowhi = i >> 1;  // 0: row g, 1: row g+8
        if (col >= ncols) continue;
        const float sc = __int_as_float((127 - sh.xn[sh.st.cols[slot][col]]) << 23);
        const float gv = G[i] * sc, uv = U[i] * sc;
        const float h = gv / (1.0f + expf(-gv)) * uv;
        const __half hi = __float2half_rn(h);
        const __half lo = __float2half_rn(h - __half2float(hi));
        if (!(fabsf(h) <= 65504.0f)) bad = 1;
        part[i & 1] += __half2float(hi) + __half2float(lo);
        const int tp = g >> 1, pos = 2 * rowhi + (g & 1);
        const long long base = ((long long)(step * 2 * ncols) * 4 + tp) * 4 + pos;
        hs[base + (long long)(2 * col) * 16] = __half_as_ushort(hi);
        hs[base + (long long)(2 * col + 1) * 16] = __half_as_ushort(lo);
    }
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
        part[0] += __shfl_xor_sync(0xffffffffu, part[0], o);
        part[1] += __shfl_xor_sync(0xffffffffu, part[1], o);
    }
    if (g == 0) {
        if (2 * t < ncols) hsum[(2 * t) * sstr + rg] = part[0];
        if (2 * t + 1 < ncols) hsum[(2 * t + 1) * sstr + rg] = part[1];
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) set_error(p.ctrl, MOE_ERR_RANGE);
}

// Partial down output of one row-group of one slot -> dpart[slot][col][rows].
__device__ void epilogue_b(const MoeParams& p, const float* rb0, int slot, int ncols, int rg, int lane) {
    const int g = lane >> 2, t = lane & 3;
    float* dp = p.dpart + (long long)slot * p.T * p.H;
    float D[8];
    red_sum(rb0, lane, D, D + 4);
    const int row0 = 16 * rg + g;
#pragma unroll
    for (int nb = 0; nb < 2; ++nb) {
        const int col = 4 * nb + t;  // virtual columns 2col (hi), 2col+1 (lo)
        if (col < ncols) {
            dp[(long long)col * p.H + row0] = D[4 * nb + 0] + D[4 * nb + 1];
            dp[(long long)col * p.H + row0 + 8] = D[4 * nb + 2] + D[4 * nb + 3];
        }
    }
}

// An epilogue warp: units r = e, e + NEPI, ... in the order the consumers
// deposit them; the 8 warps' partials are summed in warp order.  After the
// last unit: the second grid barrier, then this CTA's slice of the combine.
__device__ void epilogue_warp(const MoeParams& p, Shared& sh, float* red, int e, int sstr) {
    const int lane = threadIdx.x & 31;
    bool ok = true;
    for (int r = e;; r += NEPI) {
        const int b = r % p.nred;
        const uint32_t ph = (uint32_t)(r / p.nred) & 1u;
        if (!mbar_wait(&sh.rfull[b], ph, WAIT_LIMIT)) { ok = false; break; }
        const RedInfo ri = sh.rinfo[b];
        if (ri.kind == UNIT_END) break;
        const float* rb0 = red + b * NCW * 32 * 8;
        if (ri.kind == UNIT_A) epilogue_a(p, sh, rb0, ri.slot, ri.ncols, ri.rg, lane, sstr);
        else if (ri.kind == UNIT_B) epilogue_b(p, rb0, ri.slot, ri.ncols, ri.rg, lane);
        __syncwarp();
        if (lane == 0) {
            mbar_arrive(&sh.rempty[b]);
            if (ri.kind == UNIT_A_END) mbar_arrive(&sh.adone);   // this warp's h stores are all issued
        }
    }
    // every partial of this CTA is stored; wait for all CTAs' (second barrier)
    asm volatile("bar.sync 3, %0;" ::"n"(NEPI * 32) : "memory");
    int& bar_ok = sh.bar_ok;
    if (e == 0 && lane == 0)
        bar_ok = ok && !sh.abort_flag && grid_barrier(reinterpret_cast<unsigned long long*>(p.ctrl + MOE_CTRL_BAR_D));
    asm volatile("bar.sync 3, %0;" ::"n"(NEPI * 32) : "memory");
    if (!bar_ok) {
        if (e == 0 && lane == 0) {
            set_error(p.ctrl, MOE_ERR_TIMEOUT);
            sh.abort_flag = 1;
        }
        return;
    }
    // combine: y[c] = sum_j w[c][j] * partial[slot(c, j)] + partial[shared], in
    // the fixed order j = 0 .. k-1 then the shared expert (column c does not
    // depend on T); this CTA owns elements [n b / G, n (b+1) / G)
    const SlotTable& S = sh.st;
    const long long n = (long long)p.T * p.H;
    const int i0 = (int)(n * blockIdx.x / gridDim.x), i1 = (int)(n * (blockIdx.x + 1) / gridDim.x);
    for (int i = i0 + e * 32 + lane; i < i1; i += NEPI * 32) {
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

// ------------------------------------------------------------- consumers ---

struct RedCursor {
    int b = 0;
    uint32_t ph = 0;   // parity of the rfull phase being filled; rempty waits for ph ^ 1
};

// Deposit this warp's partials for the next reduction unit.
__device__ __forceinline__ bool red_deposit(Shared& sh, int nred, float* red, RedCursor& rc, int w, int lane,
                                            const float v[8], const RedInfo& info) {
    if (!mbar_wait(&sh.rempty[rc.b], rc.ph ^ 1u, WAIT_LIMIT)) return false;
    float* my = red + ((rc.b * NCW + w) * 2 * 32 + lane) * 4;   // [buffer][warp][half][lane][4]
    *reinterpret_cast<float4*>(my) = make_float4(v[0], v[1], v[2], v[3]);
    *reinterpret_cast<float4*>(my + 32 * 4) = make_float4(v[4], v[5], v[6], v[7]);
    if (w == 0 && lane == 0) sh.rinfo[rc.b] = info;
    __syncwarp();
    if (lane == 0) mbar_arrive(&sh.rfull[rc.b]);
    if (++rc.b == nred) { rc.b = 0; rc.ph ^= 1u; }
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
template <int FMT, bool TWO, class SRC>
__device__ __forceinline__ void stepA(const uint8_t* st, int c, int H, int lane, int g, const SRC& bs, const float* sA0,
                                      const float* sA1, AccA& ag, AccA& au) {
    const int nt = rfx_chunk_tiles(H, c);
    if (nt == 8) {
        float S0[8], S1[8];
        ld8(sA0 + 8 * c, S0);
        if (TWO) ld8(sA1 + 8 * c, S1);
        chunkA_full<FMT, TWO>(st, st + MOE_HALF_BYTES, lane, g, bs, c * 16, S0, S1, ag, au);
    } else {
        chunkA_partial<FMT, true>(st, st + MOE_HALF_BYTES, nt, lane, g, bs, c * 16, ag, au);
    }
}

// One down chunk.
template <int FMT, int NB, class SRC>
__device__ __forceinline__ void stepB(const uint8_t* st, int c, int I, int lane, int g, int t, const SRC* bs,
                                      const float* hsum, int ncols, int sstr, AccB<NB>& ab) {
    const int nt = rfx_chunk_tiles(I, c);
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
        chunkB_full<FMT, NB>(st, lane, g, bs, c * 16, Sb, ab);
    } else {
        chunkB_partial<FMT, NB>(st, nt, lane, g, bs, c * 16, ab);
    }
}

__device__ __forceinline__ int full_chunk_bytes(int fmt) { return 128 * rfx_block_bytes(fmt); }

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

__device__ __forceinline__ bool cons_next(Shared& sh, ConsRing& rp, StageRec& r) {
    if (!mbar_wait(&sh.full[rp.stage], rp.phase, WAIT_LIMIT)) return false;
    r = sh.rec[rp.stage];
    return true;
}

__device__ __forceinline__ int fmt_a(const MoeParams& p, const SlotTable& S, int slot) {
    return S.expert[slot] < 0 ? p.fsA : p.fA;
}
__device__ __forceinline__ int fmt_b(const MoeParams& p, const SlotTable& S, int slot) {
    return S.expert[slot] < 0 ? p.fsB : p.fB;
}

// Gate/up stages of one format, from the current record r (first span of a
// row-group) while the records stay gate/up spans of that format; returns with
// the next record in r.
template <int FMT, bool TWO>
__device__ __forceinline__ bool loop_a(const MoeParams& p, Shared& sh, uint8_t* ring, uint8_t* xh, float* red, ConsRing& rp,
                       RedCursor& rc, StageRec& r) {
    const SlotTable& S = sh.st;
    const int w = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int nxc = (p.has_shared && p.fsA != p.fA) ? 2 : 1;
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
            const int ci = (S.expert[slot] < 0 && nxc == 2) ? 1 : 0;
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
        if (c < nch) stepA<FMT, TWO>(ring + rp.stage * MOE_STAGE_BYTES + w * FULLB, c, p.H, lane, g, bs, sA0, sA1, ag, au);
        cons_release(p, sh, rp, w, lane);
        if (r.flags & REC_LAST) {
            float v[8];
            finishA<FMT>(ag, v);
            finishA<FMT>(au, v + 4);
            if (!red_deposit(sh, p.nred, red, rc, w, lane, v, RedInfo{UNIT_A, slot, ncols, r.rg})) return false;
        }
        if (!cons_next(sh, rp, r)) return false;
        if (r.kind != 0 || ((r.flags & REC_FIRST) && fmt_a(p, S, r.slot) != FMT)) return true;
    }
}

// Down stages of one format (one or two row-groups per stage, see the
// producer), from the current record r while the records stay down spans of
// that format; returns with the next record in r.
template <int FMT, int NB, int HSTRIDE>
__device__ __forceinline__ bool loop_b(const MoeParams& p, Shared& sh, uint8_t* ring, uint8_t* xh, int hbytes_max, float* red, int sstr,
                       ConsRing& rp, RedCursor& rc, StageRec& r) {
    const SlotTable& S = sh.st;
    const int w = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int nch = rfx_num_chunks(p.I);
    constexpr int FULLB = 128 * (FMT * 4 + (FMT == 4 ? 1 : 2));
    AccB<NB> ab;
    BSrcK<HSTRIDE> bs[NB];
    const float* hsum = (const float*)xh;
    int slot = -1, hseq = -1, ncols = 1;
    while (true) {
        const int buf_h = r.hseq & 1;
        if (r.flags & REC_HNEW) {
            if (!mbar_wait(&sh.hfull[buf_h], (r.hseq >> 1) & 1, WAIT_LIMIT)) return false;
        }
        if (r.slot != slot || r.hseq != hseq) {
            slot = r.slot;
            hseq = r.hseq;
            ncols = S.ncols[slot];
            const uint8_t* hs = xh + buf_h * hbytes_max;
            const int vst = 64 * ncols;  // bytes per k16 step
#pragma unroll
            for (int nb = 0; nb < NB; ++nb) {
                const int vv = min(8 * nb + g, 2 * ncols - 1);
                bs[nb] = BSrcK<HSTRIDE>{hs + (vv * 4 + t) * 8, vst};
            }
            hsum = (const float*)(hs + 4 * ncols * p.I);
        }
        const int c = r.c0 + w;
        // the stage's row-groups one after the other (one copy of the chunk code)
#pragma unroll 1
        for (int i = 0; i < r.n; ++i) {
            if (r.flags & REC_FIRST) ab.zero();
            if (c < nch)
                stepB<FMT, NB>(ring + rp.stage * MOE_STAGE_BYTES + i * MOE_HALF_BYTES + w * FULLB, c, p.I, lane, g, t, bs,
                               hsum, ncols, sstr, ab);
            if (r.flags & REC_LAST) {
                float vb[NB][4], v[8];
                finishB<FMT, NB>(ab, vb);
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    v[k] = vb[0][k];
                    v[4 + k] = NB > 1 ? vb[NB - 1][k] : 0.f;
                }
                if (!red_deposit(sh, p.nred, red, rc, w, lane, v, RedInfo{UNIT_B, slot, ncols, r.rg + i})) return false;
            }
        }
        cons_release(p, sh, rp, w, lane);
        if (r.flags & REC_HDONE) {
            // every stage of this slot is consumed: release its h buffer
            __syncwarp();
            if (lane == 0) mbar_arrive(&sh.hfree[buf_h]);
        }
        if (!cons_next(sh, rp, r)) return false;
        if (r.kind != 1 || fmt_b(p, S, r.slot) != FMT) return true;
    }
}

// Consumer warp: the records of a CTA's stream are all its gate/up spans, then
// all its down spans, then the end record.  Each phase runs one loop per
// format (a CTA's range usually holds one or two formats).
template <int QC>
__device__ void consumer(const MoeParams& p, Shared& sh, uint8_t* ring, uint8_t* xh, int hbytes_max, float* red,
                         int sstr) {
    constexpr bool TWO = QC >= 2;           // a second live column per lane in the gate/up output
    constexpr int NB = QC >= 3 ? 2 : 1;     // n-blocks of virtual (hi, lo) columns in the down projection
    constexpr int HSTRIDE = QC == 1 ? 64 : 0;   // bytes per k16 step of h (one column: 2 virtual x 4 lanes x 8 B)
    const SlotTable& S = sh.st;
    const int w = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    ConsRing rp;
    RedCursor rc;
    StageRec r{};
    bool ok = cons_next(sh, rp, r);
    while (ok && r.kind == 0) {
        const int f = fmt_a(p, S, r.slot);
        if (f == 2) ok = loop_a<2, TWO>(p, sh, ring, xh, red, rp, rc, r);
        else if (f == 3) ok = loop_a<3, TWO>(p, sh, ring, xh, red, rp, rc, r);
        else ok = loop_a<4, TWO>(p, sh, ring, xh, red, rp, rc, r);
    }
    // the staged x is no longer read (the h copies will overwrite it); tell
    // each epilogue warp that the gate/up phase is over
    fence_proxy_async_smem();
    const float z[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int i = 0; i < NEPI && ok; ++i)
        if (!red_deposit(sh, p.nred, red, rc, w, lane, z, RedInfo{UNIT_A_END, 0, 0, 0})) ok = false;
    while (ok && r.kind == 1) {
        const int f = fmt_b(p, S, r.slot);
        if (f == 3) ok = loop_b<3, NB, HSTRIDE>(p, sh, ring, xh, hbytes_max, red, sstr, rp, rc, r);
        else if (f == 2) ok = loop_b<2, NB, HSTRIDE>(p, sh, ring, xh, hbytes_max, red, sstr, rp, rc, r);
        else ok = loop_b<4, NB, HSTRIDE>(p, sh, ring, xh, hbytes_max, red, sstr, rp, rc, r);
    }
    if (!ok) {
        set_error(p.ctrl, MOE_ERR_TIMEOUT);
        sh.abort_flag = 1;
    }
    // one end-of-work unit for each epilogue warp
    for (int i = 0; i < NEPI; ++i) (void)red_deposit(sh, p.nred, red, rc, w, lane, z, RedInfo{UNIT_END, 0, 0, 0});
}

// x (bf16 [T][H], global) -> shared memory for the gate/up B operand: per
// column c, x * 2^xn[c] with xn[c] putting max|x| in [2^13, 2^14), times
// 2^-s_b for the tile's bit offset in the gate/up format (one copy per format
// in use), rounded to fp16 in fragment order [c][step][t][k 2t,2t+1,2t+8,2t+9];
// plus the block sums of the staged values (times 2^s_b) for the offset
// correction.  Run by `nthr` threads (sid = 0 .. nthr-1, whole warps); one item
// is one (step, t) fragment of a column, 8 consecutive items one 32-block.
// The columns (T <= MAXC) are handled side by side in each item step, so the
// per-column chains (loads, shuffles) overlap.
template <int MAXC>
__device__ void stage_x(const MoeParams& p, Shared& sh, uint8_t* xh, const uint32_t* x32, int sid, int nthr) {
    const int lane = sid & 31;
    const int per_col = p.H / 4;      // items per column
    const int hp = p.H / 2;           // bf16 pairs per column
    // pass 1: max |x| per column (a warp's items never straddle a column)
    uint32_t m[MAXC];
#pragma unroll
    for (int c = 0; c < MAXC; ++c) m[c] = 0u;
    for (int j0 = sid - lane; j0 < per_col; j0 += nthr) {
        const int j = j0 + lane;
        if (j < per_col) {
            const int step = j >> 2, tt = j & 3;
#pragma unroll
            for (int c = 0; c < MAXC; ++c)
                if (c < p.T) {
                    const uint32_t* src = x32 + (size_t)c * hp + step * 8 + tt;
                    const uint32_t v0 = src[0], v1 = src[4];
                    m[c] = max(m[c], max((v0 << 16) & 0x7fffffffu, v0 & 0x7fff0000u));
                    m[c] = max(m[c], max((v1 << 16) & 0x7fffffffu, v1 & 0x7fff0000u));
                }
        }
    }
#pragma unroll
    for (int c = 0; c < MAXC; ++c)
        if (c < p.T) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m[c] = max(m[c], __shfl_xor_sync(0xffffffffu, m[c], o));
            if (lane == 0 && m[c]) atomicMax(&sh.xmax[c], m[c]);
        }
    asm volatile("bar.sync 1, %0;" ::"r"(nthr) : "memory");
    if (sid < p.T) {
        const uint32_t mm = sh.xmax[sid];
        const int n = mm ? 13 - ((int)((mm >> 23) & 255u) - 127) : 0;
        sh.xn[sid] = max(-100, min(100, n));
    }
    asm volatile("bar.sync 1, %0;" ::"r"(nthr) : "memory");
    // pass 2: scale, round to fp16, write fragments and block sums
    const int nxc = (p.has_shared && p.fsA != p.fA) ? 2 : 1;
    float* sx = (float*)(xh + nxc * p.T * p.x_stride);
    const int sxs = moe_sxs(p.H);
    int xn[MAXC];
#pragma unroll
    for (int c = 0; c < MAXC; ++c) xn[c] = c < p.T ? sh.xn[c] : 0;
    for (int ci = 0; ci < nxc; ++ci) {
        const int fmt = ci == 0 ? p.fA : p.fsA;
        for (int j0 = sid - lane; j0 < per_col; j0 += nthr) {
            const int j = j0 + lane;
            const int step = j >> 2, tt = j & 3;
            const int sb = s_pos(fmt, step * 16, p.H);
            float sum[MAXC];
#pragma unroll
            for (int c = 0; c < MAXC; ++c) {
                sum[c] = 0.f;
                if (c < p.T && j < per_col) {
                    uint8_t* dst = xh + (ci * p.T + c) * p.x_stride;
                    const uint32_t* src = x32 + (size_t)c * hp + step * 8 + tt;
                    const uint32_t v0 = src[0], v1 = src[4];
                    const float sc = __int_as_float((127 + xn[c] - sb) << 23);
                    const __half2 h0 = __floats2half2_rn(__uint_as_float(v0 << 16) * sc, __uint_as_float(v0 & 0xffff0000u) * sc);
                    const __half2 h1 = __floats2half2_rn(__uint_as_float(v1 << 16) * sc, __uint_as_float(v1 & 0xffff0000u) * sc);
                    uint2 o;
                    o.x = *reinterpret_cast<const uint32_t*>(&h0);
                    o.y = *reinterpret_cast<const uint32_t*>(&h1);
                    *reinterpret_cast<uint2*>(dst + (step * 4 + tt) * 8) = o;
                    sum[c] = ((__low2float(h0) + __high2float(h0)) + (__low2float(h1) + __high2float(h1))) *
                             __int_as_float((127 + sb) << 23);
                }
            }
            // the 8 items of a block are 8 consecutive lanes
#pragma unroll
            for (int c = 0; c < MAXC; ++c)
                if (c < p.T) {
                    float v = sum[c];
                    v += __shfl_xor_sync(0xffffffffu, v, 1);
                    v += __shfl_xor_sync(0xffffffffu, v, 2);
                    v += __shfl_xor_sync(0xffffffffu, v, 4);
                    if ((lane & 7) == 0 && j < per_col) sx[(ci * p.T + c) * sxs + (j >> 3)] = v;
                }
        }
    }
}

// ---------------------------------------------------------------- kernel ---

template <int QC>
__global__ void __launch_bounds__(NTHREADS, 1) moe_decode_kernel(MoeParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* ring = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t* xh = ring + p.ns * MOE_STAGE_BYTES;
    float* red = (float*)(xh + p.xh_bytes);
    Shared& sh = *(Shared*)((uint8_t*)red + p.nred * NCW * 32 * 8 * sizeof(float));
    const int sstr = moe_sstr(p.I);
    const int hbytes_max = 4 * p.T * (p.I + sstr);
    const int w = threadIdx.x >> 5;
    grid_dep_launch();   // the next kernel may launch (it waits for this one before its stores)
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
        mbar_init(&sh.adone, NEPI);
        mbar_init(&sh.xload, 1);
        sh.abort_flag = 0;
        sh.consumed = 0;
        for (int c = 0; c < MOE_MAXT; ++c) sh.xmax[c] = 0u;
        fence_barrier_init();
    }
    // everything below may read what the previous kernel wrote (routing, x,
    // the workspace counters)
    grid_dep_wait();
    Routing rt{};
    if (w == WARP_PRODUCER) rt = load_routing(p);
    // x: one bulk copy into the reduction buffers (first written after the
    // staging below) when it fits and is 16-byte aligned, else read from global
    const uint32_t xbytes = (uint32_t)(p.T * p.H * 2);
    const bool xbulk = xbytes <= (uint32_t)(p.nred * NCW * 32 * 8 * 4) && (((uintptr_t)p.x & 15u) == 0);
    if (xbulk && threadIdx.x == 0) {
        mbar_arrive_expect_tx(&sh.xload, xbytes);
        bulk_g2s(red, p.x, xbytes, &sh.xload, policy_evict_first());
    }
    __syncthreads();
    // The producer warp derives the slot table and its row-groups and starts
    // streaming weights at once; every other warp stages x meanwhile.
    if (w == WARP_PRODUCER) {
        if (p.T * p.k <= 32) build_slots_small(p, sh.st, rt);
        else build_slots(p, sh.st, rt);
        if ((threadIdx.x & 31) == 0) down_units(p, sh.st.nslots, sh.ub0, sh.ub1);
        asm volatile("bar.arrive 2, %0;" ::"n"(NTHREADS) : "memory");
        if ((threadIdx.x & 31) == 0) producer(p, sh, ring);
    } else {
        const int sid = w < WARP_PRODUCER ? threadIdx.x : threadIdx.x - 32;
        if (xbulk && !mbar_wait(&sh.xload, 0, WAIT_LIMIT)) set_error(p.ctrl, MOE_ERR_TIMEOUT);
        stage_x<QC == 1 ? 1 : (QC == 2 ? 4 : MOE_MAXT)>(
            p, sh, xh, xbulk ? (const uint32_t*)red : reinterpret_cast<const uint32_t*>(p.x), sid, NTHREADS - 32);
        asm volatile("bar.sync 2, %0;" ::"n"(NTHREADS) : "memory");
        if (w == WARP_HLOAD) {
            if ((threadIdx.x & 31) == 0) h_loader(p, sh, xh, hbytes_max, sstr);
        } else if (w >= WARP_EPILOGUE0) {
            epilogue_warp(p, sh, red, w - WARP_EPILOGUE0, sstr);
        } else {
            consumer<QC>(p, sh, ring, xh, hbytes_max, red, sstr);
        }
    }
}

// Shared-memory bytes of a launch (plus 1 KB alignment slack).
size_t moe_decode_smem_bytes(int ns, int nred, int xh_bytes) {
    return 1024 + (size_t)ns * MOE_STAGE_BYTES + xh_bytes + (size_t)nred * NCW * 32 * 8 * sizeof(float) + sizeof(Shared);
}

cudaError_t moe_decode_launch(const MoeParams& p, int grid, cudaStream_t stream) {
    const size_t smem = moe_decode_smem_bytes(p.ns, p.nred, p.xh_bytes);
    // q-class: one live column per lane (T = 1), two (T <= 4), two n-blocks of
    // the down projection's virtual columns (T <= 8)
    const int qc = p.T == 1 ? 0 : (p.T <= 4 ? 1 : 2);
    auto kern = qc == 0 ? moe_decode_kernel<1> : (qc == 1 ? moe_decode_kernel<2> : moe_decode_kernel<3>);
    // the dynamic shared-memory limit, once per device and kernel
    static SmemLimit limit[3];
    cudaError_t err = limit[qc].ensure((const void*)kern, (int)smem);
    if (err != cudaSuccess) return err;
    // cooperative: every CTA is resident at once (the two grid barriers need it)
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(NTHREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute at[2];
    at[0].id = cudaLaunchAttributeCooperative;
    at[0].val.cooperative = 1;
    // programmatic dependent of the kernel before it (the router): the CTAs
    // start and set up while it finishes, and wait for it before any load
    at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 2;
    err = cudaLaunchKernelEx(&cfg, kern, p);
    return err;
}

}  // namespace rfx
