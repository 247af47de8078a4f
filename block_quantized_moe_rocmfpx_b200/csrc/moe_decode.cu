// moe_decode.cu -- MoE FFN decode / speculative-verify step on packed
// ROCmFPX-style experts, one persistent kernel per layer.
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
//  - Tasks: A = (slot, 32 gate/up rows) -> SwiGLU -> h; B = (slot, 32 down
//    rows) -> partial d.  Tasks are handed out by a global atomic counter, A
//    before B, so a B task only ever waits on A tasks already running.
//  - Per CTA: one lane of the producer warp streams packed spans of 8 chunks
//    HBM -> shared memory with 1-D bulk copies (TMA, evict-first L2 policy)
//    into a ring of stages; one lane of the h warp bulk-copies the SwiGLU
//    output h of a slot once all of its gate/up rows are published.  8 consumer warps take one
//    chunk of every stage each, decode it in registers (one AND per A
//    register, see rfx_tile.cuh) and run mma.sync m16n8k16 in fp16: x
//    normalised per column by a power of two for gate/up, an exact hi/lo fp16
//    split of h for down.  2 epilogue warps sum the 8 warps' partials of
//    each row-group in a fixed order and run SwiGLU or the combine, so the
//    consumers never wait on global-memory latency.
//  - Combine: the last down task to finish a 16-row group sums the slots'
//    partials in a fixed order (routing order j, then shared), so y does not
//    depend on scheduling and column t is bitwise the same for any T.
//  - Every wait is bounded; a timeout sets a workspace error flag and the CTA
//    drains its in-flight copies and exits.
#include <cuda_runtime.h>

#include "moe_decode.h"
#include "rfx_tile.cuh"

namespace rfx {

constexpr int NCW = 8;                       // consumer warps 0..7
constexpr int WARP_PRODUCER = NCW;           // weight bulk copies (one lane)
constexpr int WARP_HLOAD = NCW + 1;          // h bulk copies of the down tasks (one lane)
constexpr int NEPI = 2;                      // epilogue warps: reductions, SwiGLU, combine
constexpr int WARP_EPILOGUE0 = NCW + 2;
constexpr int NTHREADS = (NCW + 2 + NEPI) * 32;
constexpr int QN = 4;
constexpr int NRED_MAX = MOE_MAX_RED;        // reduction buffers: unit r -> buffer r % p.nred,
                                             // epilogue warp r % NEPI
constexpr long long WAIT_LIMIT = 4000000000LL;

struct SlotTable {
    int nslots;
    int expert[MOE_MAXS];
    int ncols[MOE_MAXS];
    signed char cols[MOE_MAXS][MOE_MAXT];
    signed char tslot[MOE_MAXT][MOE_MAXK];
    signed char tpos[MOE_MAXT][MOE_MAXK];
    float w[MOE_MAXT][MOE_MAXK];
    unsigned mask[32];
    int prefix[32];
    int idx[MOE_MAXT * MOE_MAXK];
    unsigned char ok[MOE_MAXT * MOE_MAXK];
};

struct RedInfo {
    int kind;      // 0: gate/up row-group, 1: down row-group, -1: end of work
    int slot, ncols, rg, last_of_task;
};

// What a ring stage holds, written by the producer with the stage.
enum : short { REC_FIRST = 1, REC_LAST = 2, REC_TFIRST = 4, REC_TLAST = 8 };
struct __align__(16) StageRec {
    short kind;    // 0: gate/up span, 1: down span, -1: end of work (no copy)
    short slot;
    short rg;      // row-group of the matrix (rows 16*rg ..)
    short c0;      // first chunk of the span
    short flags;   // REC_*: first / last span of the row-group, of the task
    short pad[3];
};

struct Shared {
    uint64_t full[MOE_MAX_STAGES];
    uint64_t empty[MOE_MAX_STAGES];
    uint64_t hfull[2], hfree[2];
    uint64_t xfree;
    uint64_t rfull[NRED_MAX], rempty[NRED_MAX];
    uint64_t hqf[QN], hqe[QN];
    int hq[QN];
    StageRec rec[MOE_MAX_STAGES];
    RedInfo rinfo[NRED_MAX];
    volatile int abort_flag;
    volatile int consumed;   // stages released by all consumer warps (for the abort drain)
    unsigned xmax[MOE_MAXT]; // max |x| per column (fp32 bits)
    int xn[MOE_MAXT];        // x is staged as x * 2^xn[c] (then 2^-s_b per tile position)
    SlotTable st;
};

struct Task {
    int kind, slot, rb;
};

__device__ __forceinline__ Task decode_task(int t, int nslots, int nrbA, int nrbB) {
    const int nA = nslots * nrbA;
    if (t < nA) return {0, t / nrbA, t % nrbA};
    t -= nA;
    return {1, t / nrbB, t % nrbB};
}

__device__ __forceinline__ void set_error(uint32_t* ctrl, uint32_t bits) { atomicOr(ctrl + MOE_CTRL_ERR, bits); }

__device__ void build_slots(const MoeParams& p, SlotTable& S) {
    const int lane = threadIdx.x & 31;
    const int n = p.T * p.k;
    // one coalesced read of the routing into shared memory, then work from there
    for (int i = lane; i < n; i += 32) {
        S.idx[i] = p.idx[i];
        S.w[i / p.k][i % p.k] = p.wts[i];
    }
    S.mask[lane] = 0u;
    __syncwarp();
    for (int i = lane; i < n; i += 32) {
        const int c = i / p.k, j = i % p.k;
        const int e = S.idx[i];
        bool ok = e >= 0 && e < p.E;
        if (!ok) set_error(p.ctrl, MOE_ERR_EXPERT);
        for (int jj = 0; jj < j && ok; ++jj)
            if (S.idx[c * p.k + jj] == e) { ok = false; set_error(p.ctrl, MOE_ERR_DUP); }
        S.ok[i] = ok ? 1 : 0;
        S.tslot[c][j] = -1;
        if (ok) atomicOr(&S.mask[e >> 5], 1u << (e & 31));
    }
    __syncwarp();
    const int base = p.has_shared ? 1 : 0;
    {
        int pc = __popc(S.mask[lane]);
        int incl = pc;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        S.prefix[lane] = incl - pc;
        if (lane == 31) S.nslots = base + incl;
    }
    for (int s = lane; s < MOE_MAXS; s += 32) S.ncols[s] = 0;
    __syncwarp();
    for (int i = lane; i < n; i += 32) {
        if (!S.ok[i]) continue;
        const int c = i / p.k, j = i % p.k;
        const int e = S.idx[i];
        const int s = base + S.prefix[e >> 5] + __popc(S.mask[e >> 5] & ((1u << (e & 31)) - 1u));
        // position of column c among the columns routing to e (columns ascend);
        // each earlier column counts once even if it repeats e (flagged above)
        int pos = 0;
        for (int c2 = 0; c2 < c; ++c2) {
            for (int j2 = 0; j2 < p.k; ++j2)
                if (S.idx[c2 * p.k + j2] == e) { ++pos; break; }
        }
        S.expert[s] = e;
        S.cols[s][pos] = (signed char)c;
        S.tslot[c][j] = (signed char)s;
        S.tpos[c][j] = (signed char)pos;
        atomicAdd(&S.ncols[s], 1);
    }
    if (p.has_shared && lane == 0) {
        S.expert[0] = -1;
        S.ncols[0] = p.T;
        for (int c = 0; c < p.T; ++c) S.cols[0][c] = (signed char)c;
    }
    __syncwarp();
}

// Packed stream of the A (gate, up) or B (down) matrix of a slot.
struct MatRef {
    const uint8_t* a;
    const uint8_t* b;
    int fmt;
};

__device__ __forceinline__ MatRef slot_mats(const MoeParams& p, int e, int kind) {
    if (kind == 0) {
        if (e < 0) return {p.shg, p.shu, p.fsA};
        return {p.gate + (long long)e * p.sg, p.up + (long long)e * p.su, p.fA};
    }
    if (e < 0) return {p.shd, nullptr, p.fsB};
    return {p.down + (long long)e * p.sd, nullptr, p.fB};
}

// ------------------------------------------------------------- producer ---
//
// Per task (32 rows = 2 row-groups) and per row-group, one stage per span of
// up to 8 chunks: a single bulk copy per matrix of the contiguous span.  The
// stage record (what the stage holds) is written before the arrive that
// publishes the stage, so a consumer reads it after its acquire on `full`.

__device__ void producer(const MoeParams& p, Shared& sh, uint8_t* ring) {
    const SlotTable& S = sh.st;
    const int nrbA = p.I / 32, nrbB = p.H / 32;
    const int ntasks = S.nslots * (nrbA + nrbB);
    const uint64_t pol_w = policy_evict_first();
    int stage = 0;
    uint32_t ephase = 1;          // parity to wait for on empty[stage] (fresh barriers pass)
    int sc = 0;
    bool ok = true;
    int next = (int)atomicAdd(p.ctrl + MOE_CTRL_TASK, 1u);
    int hi = 0;
    uint32_t hphase = 1;
    while (ok) {
        const int t = next;
        if (t >= ntasks) break;
        next = (int)atomicAdd(p.ctrl + MOE_CTRL_TASK, 1u);   // used next iteration: latency hidden
        const Task tk = decode_task(t, S.nslots, nrbA, nrbB);
        if (tk.kind == 1) {
            // hand the h copy of this down task to the h lane
            if (!mbar_wait(&sh.hqe[hi], hphase, WAIT_LIMIT)) { ok = false; break; }
            sh.hq[hi] = tk.slot;
            mbar_arrive(&sh.hqf[hi]);
            if (++hi == QN) { hi = 0; hphase ^= 1u; }
        }
        const int e = S.expert[tk.slot];
        const MatRef m = slot_mats(p, e, tk.kind);
        const int K = tk.kind == 0 ? p.H : p.I;
        const int nch = rfx_num_chunks(K);
        const long long rgb = rfx_rowgroup_bytes(m.fmt, K);
        const int fullb = (int)rfx_chunk_bytes(m.fmt, 8);
        const uint32_t lastb = (uint32_t)rfx_chunk_bytes(m.fmt, rfx_chunk_tiles(K, nch - 1));
        const uint8_t* srcA = m.a + (long long)(2 * tk.rb) * rgb;
        const uint8_t* srcB = tk.kind == 0 ? m.b + (long long)(2 * tk.rb) * rgb : nullptr;
        for (int rgl = 0; rgl < 2 && ok; ++rgl) {
            for (int c0 = 0; c0 < nch; c0 += MOE_CHUNKS_PER_STAGE) {
                const int c1 = min(nch, c0 + MOE_CHUNKS_PER_STAGE);
                const uint32_t bytes = (uint32_t)((c1 - 1 - c0) * fullb) + (c1 == nch ? lastb : (uint32_t)fullb);
                if (!mbar_wait(&sh.empty[stage], ephase, WAIT_LIMIT)) { ok = false; break; }
                StageRec r{};
                r.kind = (short)tk.kind;
                r.slot = (short)tk.slot;
                r.rg = (short)(2 * tk.rb + rgl);
                r.c0 = (short)c0;
                r.flags = (short)((c0 == 0 ? REC_FIRST : 0) | (c1 == nch ? REC_LAST : 0) |
                                  (rgl == 0 && c0 == 0 ? REC_TFIRST : 0) | (rgl == 1 && c1 == nch ? REC_TLAST : 0));
                sh.rec[stage] = r;
                uint8_t* dst = ring + stage * MOE_STAGE_BYTES;
                const long long off = (long long)rgl * rgb + (long long)c0 * fullb;
                if (tk.kind == 0) {
                    mbar_arrive_expect_tx(&sh.full[stage], 2 * bytes);
                    bulk_g2s(dst, srcA + off, bytes, &sh.full[stage], pol_w);
                    bulk_g2s(dst + MOE_HALF_BYTES, srcB + off, bytes, &sh.full[stage], pol_w);
                } else {
                    mbar_arrive_expect_tx(&sh.full[stage], bytes);
                    bulk_g2s(dst, srcA + off, bytes, &sh.full[stage], pol_w);
                }
                ++sc;
                if (++stage == p.ns) { stage = 0; ephase ^= 1u; }
            }
        }
    }
    // end-of-work record: a stage with no copy
    if (ok) {
        if (mbar_wait(&sh.empty[stage], ephase, WAIT_LIMIT)) {
            StageRec r{};
            r.kind = -1;
            sh.rec[stage] = r;
            mbar_arrive(&sh.full[stage]);
        } else {
            ok = false;
        }
    }
    // stop the h lane
    if (mbar_wait(&sh.hqe[hi], hphase, WAIT_LIMIT)) {
        sh.hq[hi] = -1;
        mbar_arrive(&sh.hqf[hi]);
    } else {
        ok = false;
    }
    if (!ok) {
        set_error(p.ctrl, MOE_ERR_TIMEOUT);
        sh.abort_flag = 1;
        // drain: wait (bounded) until every issued copy has landed
        for (int i = sh.consumed; i < sc; ++i) (void)mbar_wait(&sh.full[i % p.ns], (i / p.ns) & 1, WAIT_LIMIT);
    }
}

// The h lane: for each down task, in order, wait until every gate/up
// row-group of its slot is published, then bulk-copy the slot's h and its
// block sums (and nothing of the weight stream waits on this).
__device__ void h_loader(const MoeParams& p, Shared& sh, uint8_t* xh, int hbytes_max, int sstr) {
    const SlotTable& S = sh.st;
    const uint64_t pol_h = policy_evict_last();
    const uint32_t need = (uint32_t)(p.I / 16);
    int hi = 0;
    uint32_t hphase = 0;
    int bseq = 0;
    uint32_t known_ready[3] = {0u, 0u, 0u};   // slots already seen complete (bit per slot)
    bool ok = true;
    while (true) {
        if (!mbar_wait(&sh.hqf[hi], hphase, WAIT_LIMIT)) { ok = false; break; }
        const int slot = sh.hq[hi];
        mbar_arrive(&sh.hqe[hi]);
        if (++hi == QN) { hi = 0; hphase ^= 1u; }
        if (slot < 0) break;
        if (bseq == 0 && !mbar_wait(&sh.xfree, 0, WAIT_LIMIT)) { ok = false; break; }
        const int buf = bseq & 1;
        if (!mbar_wait(&sh.hfree[buf], ((bseq >> 1) + 1) & 1, WAIT_LIMIT)) { ok = false; break; }
        if (!(known_ready[slot >> 5] >> (slot & 31) & 1u)) {
            const long long t0 = clock64();
            unsigned nap = 32;
            while (ld_relaxed_gpu(p.ctrl + MOE_CTRL_SLOT + slot) < need) {
                if (clock64() - t0 > WAIT_LIMIT) { ok = false; break; }
                __nanosleep(nap);
                nap = min(nap * 2u, 256u);
            }
            if (!ok) break;
            known_ready[slot >> 5] |= 1u << (slot & 31);
        }
        fence_acq_rel_gpu();          // acquire side of the publishers' release
        fence_proxy_async_global();   // generic-proxy writes of h -> bulk-copy (async proxy) reads
        const uint32_t hb = 4u * (uint32_t)S.ncols[slot] * (uint32_t)(p.I + sstr);
        mbar_arrive_expect_tx(&sh.hfull[buf], hb);
        bulk_g2s(xh + buf * hbytes_max, p.hbuf + (long long)slot * (2LL * p.T * (p.I + sstr)), hb, &sh.hfull[buf],
                 pol_h);
        ++bseq;
    }
    if (!ok) {
        set_error(p.ctrl, MOE_ERR_TIMEOUT);
        sh.abort_flag = 1;
        for (int b = 0; b < 2 && b < bseq; ++b)
            (void)mbar_wait(&sh.hfull[(bseq - 1 - b) & 1], ((bseq - 1 - b) >> 1) & 1, WAIT_LIMIT);
    }
}

// ------------------------------------------------------------- epilogues ---

// SwiGLU of one row-group: undo the per-column x scaling, h = silu(g) * u,
// store h as an fp16 hi/lo pair in the fragment order of the down projection's
// B operand ([step][v][t'][4], v = 2*col + {0 hi, 1 lo}) and the row-group's
// sum of (hi + lo) per column (half of a 32-wide down block).
__device__ void epilogue_a(const MoeParams& p, const Shared& sh, const float* rb0, int slot, int ncols, int rg,
                           int lane, int sstr) {
    const int g = lane >> 2, t = lane & 3;
    uint16_t* hs = p.hbuf + (long long)slot * (2LL * p.T * (p.I + sstr));
    float* hsum = (float*)(hs + 2LL * ncols * p.I);
    float G[4] = {0.f, 0.f, 0.f, 0.f}, U[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int w = 0; w < NCW; ++w) {
        const float* r = rb0 + (w * 32 + lane) * 8;
#pragma unroll
        for (int i = 0; i < 4; ++i) { G[i] += r[i]; U[i] += r[4 + i]; }
    }
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

// Partial down output of one row-group -> dpart; the last slot to finish the
// row-group sums all slots' partials in a fixed order into y.
__device__ void epilogue_b(const MoeParams& p, const SlotTable& S, const float* rb0, int slot, int ncols, int rg,
                           int lane) {
    const int g = lane >> 2, t = lane & 3;
    float* dp = p.dpart + (long long)slot * p.T * p.H;
    float D[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int w = 0; w < NCW; ++w) {
        const float* r = rb0 + (w * 32 + lane) * 8;
#pragma unroll
        for (int i = 0; i < 8; ++i) D[i] += r[i];
    }
    const int row0 = 16 * rg + g;
#pragma unroll
    for (int nb = 0; nb < 2; ++nb) {
        const int col = 4 * nb + t;  // virtual columns 2col (hi), 2col+1 (lo)
        if (col < ncols) {
            dp[(long long)col * p.H + row0] = D[4 * nb + 0] + D[4 * nb + 1];
            dp[(long long)col * p.H + row0 + 8] = D[4 * nb + 2] + D[4 * nb + 3];
        }
    }
    // warp barrier, then one release/acquire atomic for the whole warp's stores
    __syncwarp();
    uint32_t prev = 0;
    if (lane == 0) prev = atom_add_acq_rel_gpu(p.ctrl + MOE_CTRL_ROWBLK + rg, 1u);
    prev = __shfl_sync(0xffffffffu, prev, 0);
    if (prev != (uint32_t)S.nslots - 1) return;
    __syncwarp();   // lane 0's acquire orders the other lanes' reads of dpart below
    for (int it = lane; it < 16 * p.T; it += 32) {
        const int row = 16 * rg + (it & 15), c = it >> 4;
        float acc = 0.f;
        for (int j = 0; j < p.k; ++j) {
            const int s2 = S.tslot[c][j];
            if (s2 < 0) continue;
            const float v = __ldcg(p.dpart + ((long long)s2 * p.T + S.tpos[c][j]) * p.H + row);
            acc = fmaf(S.w[c][j], v, acc);
        }
        if (p.has_shared) acc += __ldcg(p.dpart + (long long)c * p.H + row);
        p.y[(long long)c * p.H + row] = acc;
    }
    __syncwarp();
    if (lane == 0) p.ctrl[MOE_CTRL_ROWBLK + rg] = 0u;
}

// An epilogue warp: units r = e, e + NEPI, ... in the order the consumers
// deposit them; the 8 warps' partials are summed in warp order.
__device__ void epilogue_warp(const MoeParams& p, Shared& sh, float* red, int e, int sstr) {
    const int lane = threadIdx.x & 31;
    for (int r = e;; r += NEPI) {
        const int b = r % p.nred;
        const uint32_t ph = (uint32_t)(r / p.nred) & 1u;
        if (!mbar_wait(&sh.rfull[b], ph, WAIT_LIMIT)) {
            set_error(p.ctrl, MOE_ERR_TIMEOUT);
            sh.abort_flag = 1;
            break;
        }
        const RedInfo ri = sh.rinfo[b];
        if (ri.kind < 0) break;
        const float* rb0 = red + b * NCW * 32 * 8;
        if (ri.kind == 0) {
            epilogue_a(p, sh, rb0, ri.slot, ri.ncols, ri.rg, lane, sstr);
            // this row-group of h is complete: publish it to the down tasks
            // (the bulk-copy reader fences the async proxy after its acquire)
            __syncwarp();
            if (lane == 0) red_add_release_gpu(p.ctrl + MOE_CTRL_SLOT + ri.slot, 1u);
        } else {
            epilogue_b(p, sh.st, rb0, ri.slot, ri.ncols, ri.rg, lane);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.rempty[b]);
    }
}

// ------------------------------------------------------------- consumers ---

struct RedCursor {
    int b = 0;
    uint32_t ph = 0;   // parity of the rfull phase being filled; rempty waits for ph ^ 1
};

// Deposit this warp's partials for the next reduction unit.
__device__ __forceinline__ bool red_deposit(const MoeParams& p, Shared& sh, float* red, RedCursor& rc, int w, int lane,
                                            const float v[8], const RedInfo& info) {
    if (!mbar_wait(&sh.rempty[rc.b], rc.ph ^ 1u, WAIT_LIMIT)) return false;
    float* my = red + ((rc.b * NCW + w) * 32 + lane) * 8;
    *reinterpret_cast<float4*>(my) = make_float4(v[0], v[1], v[2], v[3]);
    *reinterpret_cast<float4*>(my + 4) = make_float4(v[4], v[5], v[6], v[7]);
    if (w == 0 && lane == 0) sh.rinfo[rc.b] = info;
    __syncwarp();
    if (lane == 0) mbar_arrive(&sh.rfull[rc.b]);
    if (++rc.b == p.nred) { rc.b = 0; rc.ph ^= 1u; }
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

// Ring position of a consumer warp.
struct Ring {
    int stage = 0, cc = 0;
    uint32_t fphase = 0;
    __device__ __forceinline__ void release(const MoeParams& p, Shared& sh, int w, int lane) {
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.empty[stage]);
        ++cc;
        if (w == 0 && lane == 0) sh.consumed = cc;
        if (++stage == p.ns) { stage = 0; fphase ^= 1u; }
    }
};

__device__ __forceinline__ void ld8(const float* src, float d[8]) {
    const float4 a = ldsf4((const uint8_t*)src), b = ldsf4((const uint8_t*)(src + 4));
    d[0] = a.x; d[1] = a.y; d[2] = a.z; d[3] = a.w;
    d[4] = b.x; d[5] = b.y; d[6] = b.z; d[7] = b.w;
}

// One gate/up chunk pair (chunk c of the stage's span, this warp's share).
template <int FMT, bool TWO>
__device__ __forceinline__ void stepA(const uint8_t* st, int c, int H, int lane, int g, const BSrc& bs, const float* sA0,
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
template <int FMT, int NB>
__device__ __forceinline__ void stepB(const uint8_t* st, int c, int I, int lane, int g, int t, const BSrc* bs,
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

// Consumer warp: one flat loop over the ring.  Every CTA's stream holds all of
// its gate/up spans before its down spans (tasks are handed out A first), so
// the two phases are two loops with their own accumulators.
template <int QC>
__device__ void consumer(const MoeParams& p, Shared& sh, uint8_t* ring, uint8_t* xh, int hbytes_max, float* red,
                         int sstr) {
    constexpr bool TWO = QC >= 2;           // a second live column per lane in the gate/up output
    constexpr int NB = QC >= 3 ? 2 : 1;     // n-blocks of virtual (hi, lo) columns in the down projection
    const SlotTable& S = sh.st;
    const int w = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int nxc = (p.has_shared && p.fsA != p.fA) ? 2 : 1;
    const float* sx = (const float*)(xh + nxc * p.T * p.x_stride);   // [copy][col][sxs]
    const int sxs = moe_sxs(p.H);
    const int nchA = rfx_num_chunks(p.H), nchB = rfx_num_chunks(p.I);
    Ring ring_pos;
    RedCursor rc;
    bool ok = true;
    StageRec r{};
    // ---- gate/up spans -> SwiGLU partials
    {
        AccA ag, au;
        ag.zero();
        au.zero();
        BSrc bs{xh, 0, false};
        const float* sA0 = sx;
        const float* sA1 = sx;
        int slot = 0, ncols = 0, fmt = 2;
        while (true) {
            if (!mbar_wait(&sh.full[ring_pos.stage], ring_pos.fphase, WAIT_LIMIT)) { ok = false; break; }
            r = sh.rec[ring_pos.stage];
            if (r.kind != 0) break;
            if (r.flags & REC_FIRST) {
                slot = r.slot;
                const int e = S.expert[slot];
                ncols = S.ncols[slot];
                fmt = e < 0 ? p.fsA : p.fA;
                const int ci = (e < 0 && nxc == 2) ? 1 : 0;
                const int col0 = g < ncols ? S.cols[slot][g] : 0;
                bs = BSrc{xh + (ci * p.T + col0) * p.x_stride + t * 8, 32, g < ncols};
                const int c0 = 2 * t < ncols ? S.cols[slot][2 * t] : 0;
                const int c1 = 2 * t + 1 < ncols ? S.cols[slot][2 * t + 1] : 0;
                sA0 = sx + (ci * p.T + c0) * sxs;
                sA1 = sx + (ci * p.T + c1) * sxs;
                ag.zero();
                au.zero();
            }
            const int c = r.c0 + w;
            if (c < nchA) {
                const uint8_t* st = ring + ring_pos.stage * MOE_STAGE_BYTES + w * full_chunk_bytes(fmt);
                if (fmt == 2) stepA<2, TWO>(st, c, p.H, lane, g, bs, sA0, sA1, ag, au);
                else if (fmt == 3) stepA<3, TWO>(st, c, p.H, lane, g, bs, sA0, sA1, ag, au);
                else stepA<4, TWO>(st, c, p.H, lane, g, bs, sA0, sA1, ag, au);
            }
            ring_pos.release(p, sh, w, lane);
            if (r.flags & REC_LAST) {
                float v[8];
                if (fmt == 2) { finishA<2>(ag, v); finishA<2>(au, v + 4); }
                else if (fmt == 3) { finishA<3>(ag, v); finishA<3>(au, v + 4); }
                else { finishA<4>(ag, v); finishA<4>(au, v + 4); }
                const RedInfo info{0, slot, ncols, r.rg, (r.flags & REC_TLAST) ? 1 : 0};
                if (!red_deposit(p, sh, red, rc, w, lane, v, info)) { ok = false; break; }
            }
        }
    }
    // ---- down spans -> partial outputs
    if (ok && r.kind == 1) {
        // the staged x is no longer read: the h lane may overwrite it
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.xfree);
        AccB<NB> ab;
        ab.zero();
        BSrc bs[NB];
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) bs[nb] = BSrc{xh, 0, false};
        const float* hsum = (const float*)xh;
        int bseq = 0, slot = 0, ncols = 0, fmt = 3;
        while (true) {
            const int buf_h = bseq & 1;
            if (r.flags & REC_TFIRST) {
                if (!mbar_wait(&sh.hfull[buf_h], (bseq >> 1) & 1, WAIT_LIMIT)) { ok = false; break; }
            }
            if (r.flags & REC_FIRST) {
                slot = r.slot;
                const int e = S.expert[slot];
                ncols = S.ncols[slot];
                fmt = e < 0 ? p.fsB : p.fB;
                const uint8_t* hs = xh + buf_h * hbytes_max;
                const int vst = 64 * ncols;  // bytes per k16 step
#pragma unroll
                for (int nb = 0; nb < NB; ++nb) {
                    const int vv = 8 * nb + g;
                    bs[nb] = BSrc{hs + (vv * 4 + t) * 8, vst, vv < 2 * ncols};
                }
                hsum = (const float*)(hs + 4 * ncols * p.I);
                ab.zero();
            }
            const int c = r.c0 + w;
            if (c < nchB) {
                const uint8_t* st = ring + ring_pos.stage * MOE_STAGE_BYTES + w * full_chunk_bytes(fmt);
                if (fmt == 3) stepB<3, NB>(st, c, p.I, lane, g, t, bs, hsum, ncols, sstr, ab);
                else if (fmt == 2) stepB<2, NB>(st, c, p.I, lane, g, t, bs, hsum, ncols, sstr, ab);
                else stepB<4, NB>(st, c, p.I, lane, g, t, bs, hsum, ncols, sstr, ab);
            }
            ring_pos.release(p, sh, w, lane);
            if (r.flags & REC_LAST) {
                float vb[NB][4];
                if (fmt == 3) finishB<3, NB>(ab, vb);
                else if (fmt == 2) finishB<2, NB>(ab, vb);
                else finishB<4, NB>(ab, vb);
                float v[8];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    v[i] = vb[0][i];
                    v[4 + i] = NB > 1 ? vb[NB - 1][i] : 0.f;
                }
                const RedInfo info{1, slot, ncols, r.rg, (r.flags & REC_TLAST) ? 1 : 0};
                if (!red_deposit(p, sh, red, rc, w, lane, v, info)) { ok = false; break; }
            }
            if (r.flags & REC_TLAST) {
                // every span of this down task is consumed: release its h buffer
                __syncwarp();
                if (lane == 0) mbar_arrive(&sh.hfree[buf_h]);
                ++bseq;
            }
            if (!mbar_wait(&sh.full[ring_pos.stage], ring_pos.fphase, WAIT_LIMIT)) { ok = false; break; }
            r = sh.rec[ring_pos.stage];
            if (r.kind != 1) break;
        }
    }
    if (!ok) {
        set_error(p.ctrl, MOE_ERR_TIMEOUT);
        sh.abort_flag = 1;
    }
    // one end-of-work unit for each epilogue warp
    const RedInfo fin{-1, 0, 0, 0, 0};
    const float z[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int i = 0; i < NEPI; ++i) (void)red_deposit(p, sh, red, rc, w, lane, z, fin);
}

// x (bf16 [T][H], global) -> shared memory for the gate/up B operand: per
// column c, x * 2^xn[c] with xn[c] putting max|x| in [2^13, 2^14), times
// 2^-s_b for the tile's bit offset in the gate/up format (one copy per format
// in use), rounded to fp16 in fragment order [c][step][t][k 2t,2t+1,2t+8,2t+9];
// plus the block sums of the staged values (times 2^s_b) for the offset
// correction.  Run by `nthr` threads (sid = 0 .. nthr-1, whole warps); one item
// is one (step, t) fragment of a column, 8 consecutive items one 32-block.
__device__ void stage_x(const MoeParams& p, Shared& sh, uint8_t* xh, int sid, int nthr) {
    const uint32_t* x32 = reinterpret_cast<const uint32_t*>(p.x);
    const int lane = sid & 31;
    const int per_col = p.H / 4;      // items per column
    const int hp = p.H / 2;           // bf16 pairs per column
    // pass 1: max |x| per column (a warp's items never straddle a column)
    for (int c = 0; c < p.T; ++c) {
        uint32_t m = 0u;
        for (int j0 = sid - lane; j0 < per_col; j0 += nthr) {
            const int j = j0 + lane;
            if (j < per_col) {
                const int step = j >> 2, tt = j & 3;
                const uint32_t* src = x32 + (size_t)c * hp + step * 8 + tt;
                const uint32_t v0 = __ldg(src), v1 = __ldg(src + 4);
                m = max(m, max((v0 << 16) & 0x7fffffffu, v0 & 0x7fff0000u));
                m = max(m, max((v1 << 16) & 0x7fffffffu, v1 & 0x7fff0000u));
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (lane == 0 && m) atomicMax(&sh.xmax[c], m);
    }
    asm volatile("bar.sync 1, %0;" ::"r"(nthr) : "memory");
    if (sid < p.T) {
        const uint32_t m = sh.xmax[sid];
        const int n = m ? 13 - ((int)((m >> 23) & 255u) - 127) : 0;
        sh.xn[sid] = max(-100, min(100, n));
    }
    asm volatile("bar.sync 1, %0;" ::"r"(nthr) : "memory");
    // pass 2: scale, round to fp16, write fragments and block sums
    const int nxc = (p.has_shared && p.fsA != p.fA) ? 2 : 1;
    float* sx = (float*)(xh + nxc * p.T * p.x_stride);
    const int sxs = moe_sxs(p.H);
    for (int ci = 0; ci < nxc; ++ci) {
        const int fmt = ci == 0 ? p.fA : p.fsA;
        for (int c = 0; c < p.T; ++c) {
            const int xn = sh.xn[c];
            uint8_t* dst = xh + (ci * p.T + c) * p.x_stride;
            for (int j0 = sid - lane; j0 < per_col; j0 += nthr) {
                const int j = j0 + lane;
                float sum = 0.f;
                if (j < per_col) {
                    const int step = j >> 2, tt = j & 3;
                    const uint32_t* src = x32 + (size_t)c * hp + step * 8 + tt;
                    const uint32_t v0 = __ldg(src), v1 = __ldg(src + 4);
                    const int sb = s_pos(fmt, step * 16, p.H);
                    const float sc = __int_as_float((127 + xn - sb) << 23);
                    const __half2 h0 = __floats2half2_rn(__uint_as_float(v0 << 16) * sc, __uint_as_float(v0 & 0xffff0000u) * sc);
                    const __half2 h1 = __floats2half2_rn(__uint_as_float(v1 << 16) * sc, __uint_as_float(v1 & 0xffff0000u) * sc);
                    uint2 o;
                    o.x = *reinterpret_cast<const uint32_t*>(&h0);
                    o.y = *reinterpret_cast<const uint32_t*>(&h1);
                    *reinterpret_cast<uint2*>(dst + (step * 4 + tt) * 8) = o;
                    sum = ((__low2float(h0) + __high2float(h0)) + (__low2float(h1) + __high2float(h1))) *
                          __int_as_float((127 + sb) << 23);
                }
                // the 8 items of a block are 8 consecutive lanes
                sum += __shfl_xor_sync(0xffffffffu, sum, 1);
                sum += __shfl_xor_sync(0xffffffffu, sum, 2);
                sum += __shfl_xor_sync(0xffffffffu, sum, 4);
                if ((lane & 7) == 0 && j < per_col) sx[(ci * p.T + c) * sxs + (j >> 3)] = sum;
            }
        }
    }
}

template <int QC>
__global__ void __launch_bounds__(NTHREADS, 1) moe_decode_kernel(MoeParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* base = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t* ring = base;
    uint8_t* xh = ring + p.ns * MOE_STAGE_BYTES;
    float* red = (float*)(xh + p.xh_bytes);
    Shared& sh = *(Shared*)((uint8_t*)red + p.nred * NCW * 32 * 8 * sizeof(float));
    const int sstr = moe_sstr(p.I);
    const int hbytes_max = 4 * p.T * (p.I + sstr);
    const int w = threadIdx.x >> 5;

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
        mbar_init(&sh.xfree, NCW);
        for (int i = 0; i < QN; ++i) {
            mbar_init(&sh.hqf[i], 1);
            mbar_init(&sh.hqe[i], 1);
        }
        sh.abort_flag = 0;
        sh.consumed = 0;
        for (int c = 0; c < MOE_MAXT; ++c) sh.xmax[c] = 0u;
        fence_barrier_init();
    }
    __syncthreads();
    // The producer warp derives the slot table and starts streaming weights at
    // once; every other warp stages x meanwhile, then waits for the table.
    if (w == WARP_PRODUCER) {
        build_slots(p, sh.st);
        asm volatile("bar.arrive 2, %0;" ::"n"(NTHREADS) : "memory");
        if ((threadIdx.x & 31) == 0) producer(p, sh, ring);
    } else {
        const int sid = w < WARP_PRODUCER ? threadIdx.x : threadIdx.x - 32;
        stage_x(p, sh, xh, sid, NTHREADS - 32);
        asm volatile("bar.sync 2, %0;" ::"n"(NTHREADS) : "memory");
        if (w == WARP_HLOAD) {
            if ((threadIdx.x & 31) == 0) h_loader(p, sh, xh, hbytes_max, sstr);
        } else if (w >= WARP_EPILOGUE0) {
            epilogue_warp(p, sh, red, w - WARP_EPILOGUE0, sstr);
        } else {
            consumer<QC>(p, sh, ring, xh, hbytes_max, red, sstr);
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        const uint32_t prev = atom_add_acq_rel_gpu(p.ctrl + MOE_CTRL_EXIT, 1u);
        if (prev == gridDim.x - 1) {
            // last CTA out: reset the counters for the next call on this workspace
            for (int s = 0; s < sh.st.nslots; ++s) p.ctrl[MOE_CTRL_SLOT + s] = 0u;
            p.ctrl[MOE_CTRL_TASK] = 0u;
            __threadfence();
            p.ctrl[MOE_CTRL_EXIT] = 0u;
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
    auto kern = p.T == 1 ? moe_decode_kernel<1> : (p.T <= 4 ? moe_decode_kernel<2> : moe_decode_kernel<3>);
    // raise the dynamic shared-memory limit once (not a stream operation, so
    // it stays out of any graph capture after the first call)
    static int set_bytes[64][3] = {{0}};
    const int qc = p.T == 1 ? 0 : (p.T <= 4 ? 1 : 2);
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev >= 64 || set_bytes[dev][qc] < (int)smem) {
        err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (err != cudaSuccess) return err;
        if (dev < 64) set_bytes[dev][qc] = (int)smem;
    }
    kern<<<grid, NTHREADS, smem, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace rfx
