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
//  - Per CTA: one producer warp streams packed chunks HBM -> shared memory with
//    1-D bulk copies (TMA, evict-first L2 policy) into per-warp stage rings;
//    8 consumer warps (2 row-groups x 4 K-quarters) decode in registers and
//    run mma.sync m16n8k16 (bf16 x for gate/up, fp16 hi/lo split of h for
//    down).  K-quarter partials are reduced in shared memory by the last warp
//    to arrive, in a fixed order.
//  - Combine: the last B task to finish a 32-row block sums the slots'
//    partials in a fixed order (routing order j, then shared), so y does not
//    depend on scheduling and column t is bitwise the same for any T.
//  - Every wait is bounded; a timeout sets a workspace error flag and the CTA
//    drains its in-flight copies and exits.
#include <cuda_runtime.h>

#include "moe_decode.h"
#include "rfx_tile.cuh"

namespace rfx {

constexpr int NCW = 8;
constexpr int NTHREADS = (NCW + 1) * 32;
constexpr int QN = 4;
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
};

struct Shared {
    uint64_t full[MOE_MAX_STAGES];
    uint64_t empty[MOE_MAX_STAGES];
    uint64_t tqf[QN], tqe[QN];
    uint64_t hfull[2], hfree[2];
    uint64_t xfree;
    int tq[QN];
    int rcnt[2];
    volatile int repoch[2];
    volatile int abort_flag;
    volatile int consumed;   // stages released by all consumer warps (for the abort drain)
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
    if (lane < 32) S.mask[lane] = 0u;
    __syncwarp();
    for (int i = lane; i < n; i += 32) {
        const int c = i / p.k, j = i % p.k;
        int e = p.idx[i];
        bool ok = e >= 0 && e < p.E;
        if (!ok) set_error(p.ctrl, MOE_ERR_EXPERT);
        for (int jj = 0; jj < j && ok; ++jj)
            if (p.idx[c * p.k + jj] == e) { ok = false; set_error(p.ctrl, MOE_ERR_DUP); }
        S.w[c][j] = p.wts[i];
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
    __syncwarp();
    for (int s = lane; s < MOE_MAXS; s += 32) S.ncols[s] = 0;
    __syncwarp();
    for (int i = lane; i < n; i += 32) {
        const int c = i / p.k, j = i % p.k;
        const int e = p.idx[i];
        bool ok = e >= 0 && e < p.E;
        for (int jj = 0; jj < j && ok; ++jj)
            if (p.idx[c * p.k + jj] == e) ok = false;
        if (!ok) continue;
        const int s = base + S.prefix[e >> 5] + __popc(S.mask[e >> 5] & ((1u << (e & 31)) - 1u));
        // position of column c among the columns routing to e (columns ascend);
        // each earlier column counts once even if it repeats e (flagged above)
        int pos = 0;
        for (int c2 = 0; c2 < c; ++c2) {
            for (int j2 = 0; j2 < p.k; ++j2)
                if (p.idx[c2 * p.k + j2] == e) { ++pos; break; }
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
// up to 8 chunks: a single bulk copy per matrix of the contiguous span.

__device__ void producer(const MoeParams& p, Shared& sh, uint8_t* ring, uint8_t* xh, int hbytes_max) {
    const SlotTable& S = sh.st;
    const int nrbA = p.I / 32, nrbB = p.H / 32;
    const int ntasks = S.nslots * (nrbA + nrbB);
    const uint64_t pol_w = policy_evict_first();
    const uint64_t pol_h = policy_evict_last();
    int sc = 0, bseq = 0;
    bool ok = true;
    int next = (int)atomicAdd(p.ctrl + MOE_CTRL_TASK, 1u);
    for (int n = 0; ok; ++n) {
        int t = next;
        if (t >= ntasks) t = -1;
        else next = (int)atomicAdd(p.ctrl + MOE_CTRL_TASK, 1u);   // overlaps with this task's copies
        const int qi = n % QN;
        if (!mbar_wait(&sh.tqe[qi], ((n / QN) + 1) & 1, WAIT_LIMIT)) { ok = false; break; }
        sh.tq[qi] = t;
        mbar_arrive(&sh.tqf[qi]);
        if (t < 0) break;
        const Task tk = decode_task(t, S.nslots, nrbA, nrbB);
        const int e = S.expert[tk.slot];
        const MatRef m = slot_mats(p, e, tk.kind);
        const int K = tk.kind == 0 ? p.H : p.I;
        const int nch = rfx_num_chunks(K);
        const long long rgb = rfx_rowgroup_bytes(m.fmt, K);
        const int fullb = (int)rfx_chunk_bytes(m.fmt, 8);
        if (tk.kind == 1) {
            if (bseq == 0 && !mbar_wait(&sh.xfree, 0, WAIT_LIMIT)) { ok = false; break; }
            const int buf = bseq & 1;
            if (!mbar_wait(&sh.hfree[buf], ((bseq >> 1) + 1) & 1, WAIT_LIMIT)) { ok = false; break; }
            const uint32_t need = (uint32_t)nrbA;
            const long long t0 = clock64();
            while (ld_acquire_gpu(p.ctrl + MOE_CTRL_SLOT + tk.slot) < need) {
                if (clock64() - t0 > WAIT_LIMIT) { ok = false; break; }
                __nanosleep(32);
            }
            if (!ok) break;
            fence_proxy_async_global();
            const uint32_t hb = 4u * (uint32_t)S.ncols[tk.slot] * (uint32_t)p.I;
            mbar_arrive_expect_tx(&sh.hfull[buf], hb);
            bulk_g2s(xh + buf * hbytes_max, p.hbuf + (long long)tk.slot * (2LL * p.T * p.I), hb, &sh.hfull[buf],
                     pol_h);
            ++bseq;
        }
        for (int rgl = 0; rgl < 2 && ok; ++rgl) {
            const long long rgoff = (long long)(2 * tk.rb + rgl) * rgb;
            for (int c0 = 0; c0 < nch; c0 += MOE_CHUNKS_PER_STAGE) {
                const int c1 = min(nch, c0 + MOE_CHUNKS_PER_STAGE);
                // bytes of chunks [c0, c1): full chunks plus a possibly partial last one
                const uint32_t bytes = (uint32_t)((c1 - 1 - c0) * fullb + rfx_chunk_bytes(m.fmt, rfx_chunk_tiles(K, c1 - 1)));
                const int s = sc % p.ns;
                if (!mbar_wait(&sh.empty[s], ((sc / p.ns) + 1) & 1, WAIT_LIMIT)) { ok = false; break; }
                uint8_t* dst = ring + s * MOE_STAGE_BYTES;
                const long long off = rgoff + (long long)c0 * fullb;
                if (tk.kind == 0) {
                    mbar_arrive_expect_tx(&sh.full[s], 2 * bytes);
                    bulk_g2s(dst, m.a + off, bytes, &sh.full[s], pol_w);
                    bulk_g2s(dst + MOE_HALF_BYTES, m.b + off, bytes, &sh.full[s], pol_w);
                } else {
                    mbar_arrive_expect_tx(&sh.full[s], bytes);
                    bulk_g2s(dst, m.a + off, bytes, &sh.full[s], pol_w);
                }
                ++sc;
            }
        }
    }
    if (!ok) {
        set_error(p.ctrl, MOE_ERR_TIMEOUT);
        sh.abort_flag = 1;
        // drain: wait (bounded) until every issued copy has landed
        for (int i = sh.consumed; i < sc; ++i) (void)mbar_wait(&sh.full[i % p.ns], (i / p.ns) & 1, WAIT_LIMIT);
        for (int b = 0; b < 2 && b < bseq; ++b)
            (void)mbar_wait(&sh.hfull[(bseq - 1 - b) & 1], ((bseq - 1 - b) >> 1) & 1, WAIT_LIMIT);
        for (int qi = 0; qi < QN; ++qi) {
            sh.tq[qi] = -1;
            mbar_arrive(&sh.tqf[qi]);
        }
    }
}

// ------------------------------------------------------------- consumers ---

// The last of the NCW warps to deposit its partial sums for row-group unit r
// returns true (and must call red_release afterwards).
__device__ __forceinline__ bool red_deposit(Shared& sh, float* red, int r, int w, int lane, const float v[8],
                                            bool& ok) {
    const int rbuf = r & 1;
    {
        const long long t0 = clock64();
        while (sh.repoch[rbuf] != r - 2) {
            if (clock64() - t0 > WAIT_LIMIT) { ok = false; return false; }
        }
    }
    float* my = red + ((rbuf * NCW + w) * 32 + lane) * 8;
#pragma unroll
    for (int i = 0; i < 8; ++i) my[i] = v[i];
    __threadfence_block();
    __syncwarp();
    int old = 0;
    if (lane == 0) old = atomicAdd(&sh.rcnt[rbuf], 1);
    old = __shfl_sync(0xffffffffu, old, 0);
    if (old != NCW - 1) return false;
    __threadfence_block();
    return true;
}

__device__ __forceinline__ void red_release(Shared& sh, int r, int lane) {
    __syncwarp();
    if (lane == 0) {
        sh.rcnt[r & 1] = 0;
        __threadfence_block();
        sh.repoch[r & 1] = r;
    }
    __syncwarp();
}

// SwiGLU of one row-group -> h (fp16 hi/lo pair per value) in the fragment
// order of the down projection's B operand: [step][v][t'][4].
__device__ void epilogue_a(const MoeParams& p, const float* rb0, int slot, int ncols, int rg, int lane) {
    const int g = lane >> 2, t = lane & 3;
    uint16_t* hs = p.hbuf + (long long)slot * (2LL * p.T * p.I);
    float G[4] = {0.f, 0.f, 0.f, 0.f}, U[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int w = 0; w < NCW; ++w) {
        const float* r = rb0 + (w * 32 + lane) * 8;
#pragma unroll
        for (int i = 0; i < 4; ++i) { G[i] += r[i]; U[i] += r[4 + i]; }
    }
    uint32_t bad = 0;
    const int step = rg;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int col = 2 * t + (i & 1);
        const int rowhi = i >> 1;  // 0: row g, 1: row g+8
        if (col >= ncols) continue;
        const float gv = G[i];
        const float h = gv / (1.0f + expf(-gv)) * U[i];
        const __half hi = __float2half_rn(h);
        const __half lo = __float2half_rn(h - __half2float(hi));
        if (!(fabsf(h) <= 65504.0f)) bad = 1;
        const int tp = g >> 1, pos = 2 * rowhi + (g & 1);
        const long long base = ((long long)(step * 2 * ncols) * 4 + tp) * 4 + pos;
        hs[base + (long long)(2 * col) * 16] = __half_as_ushort(hi);
        hs[base + (long long)(2 * col + 1) * 16] = __half_as_ushort(lo);
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
    __threadfence();
    __syncwarp();
    uint32_t prev = 0;
    if (lane == 0) prev = atom_add_acq_rel_gpu(p.ctrl + MOE_CTRL_ROWBLK + rg, 1u);
    prev = __shfl_sync(0xffffffffu, prev, 0);
    if (prev != (uint32_t)S.nslots - 1) return;
    __threadfence();
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

__device__ void consumer(const MoeParams& p, Shared& sh, uint8_t* ring, uint8_t* xh, int hbytes_max, float* red) {
    const SlotTable& S = sh.st;
    const int w = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int nrbA = p.I / 32, nrbB = p.H / 32;
    int cc = 0, bseq = 0, r = 0;
    bool first_b = true, ok = true;
    for (int n = 0; ok; ++n) {
        const int qi = n % QN;
        if (!mbar_wait(&sh.tqf[qi], (n / QN) & 1, WAIT_LIMIT)) { ok = false; break; }
        const int task = sh.tq[qi];
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.tqe[qi]);
        if (task < 0 || sh.abort_flag) break;
        const Task tk = decode_task(task, S.nslots, nrbA, nrbB);
        const int slot = tk.slot;
        const int e = S.expert[slot];
        const int ncols = S.ncols[slot];
        const int K = tk.kind == 0 ? p.H : p.I;
        const int fmt = tk.kind == 0 ? (e < 0 ? p.fsA : p.fA) : (e < 0 ? p.fsB : p.fB);
        const int fullb = (int)rfx_chunk_bytes(fmt, 8);
        const int nch = rfx_num_chunks(K);
        const int buf_h = bseq & 1;
        if (tk.kind == 1) {
            if (first_b) {
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sh.xfree);
                first_b = false;
            }
            if (!mbar_wait(&sh.hfull[buf_h], (bseq >> 1) & 1, WAIT_LIMIT)) { ok = false; break; }
        }
        BSrc bs[2];
        if (tk.kind == 0) {
            const int col = g < ncols ? S.cols[slot][g] : 0;
            bs[0] = {xh + col * p.x_stride + t * 8, 32, g < ncols};
            bs[1] = bs[0];
        } else {
            const uint8_t* hs = xh + buf_h * hbytes_max;
            const int vst = 64 * ncols;  // bytes per k16 step
#pragma unroll
            for (int nb = 0; nb < 2; ++nb) {
                const int v = 8 * nb + g;
                bs[nb] = {hs + (v * 4 + t) * 8, vst, v < 2 * ncols};
            }
        }
        const bool two_nb = tk.kind == 1 && ncols > 4;
        for (int rgl = 0; rgl < 2 && ok; ++rgl) {
            Acc<1> a0, a1;
            Acc<2> d2;
            a0.zero(); a1.zero(); d2.zero();
            for (int c0 = 0; c0 < nch; c0 += MOE_CHUNKS_PER_STAGE) {
                const int s = cc % p.ns;
                if (!mbar_wait(&sh.full[s], (cc / p.ns) & 1, WAIT_LIMIT)) { ok = false; break; }
                const int c = c0 + w;
                if (c < nch) {
                    const uint8_t* st = ring + s * MOE_STAGE_BYTES + w * fullb;
                    const int nt = rfx_chunk_tiles(K, c);
                    const int step0 = c * 16;
                    if (tk.kind == 0) {
                        switch (fmt) {
                            case 2: chunk_any2<2, false, 1>(st, st + MOE_HALF_BYTES, nt, lane, g, bs, step0, a0, a1); break;
                            case 3: chunk_any2<3, false, 1>(st, st + MOE_HALF_BYTES, nt, lane, g, bs, step0, a0, a1); break;
                            default: chunk_any2<4, false, 1>(st, st + MOE_HALF_BYTES, nt, lane, g, bs, step0, a0, a1); break;
                        }
                    } else if (!two_nb) {
                        switch (fmt) {
                            case 2: chunk_any<2, true, 1>(st, nt, lane, g, bs, step0, a0); break;
                            case 3: chunk_any<3, true, 1>(st, nt, lane, g, bs, step0, a0); break;
                            default: chunk_any<4, true, 1>(st, nt, lane, g, bs, step0, a0); break;
                        }
                    } else {
                        switch (fmt) {
                            case 2: chunk_any<2, true, 2>(st, nt, lane, g, bs, step0, d2); break;
                            case 3: chunk_any<3, true, 2>(st, nt, lane, g, bs, step0, d2); break;
                            default: chunk_any<4, true, 2>(st, nt, lane, g, bs, step0, d2); break;
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&sh.empty[s]);
                ++cc;
                if (w == 0 && lane == 0) sh.consumed = cc;
            }
            if (!ok) break;
            float v[8];
            if (tk.kind == 0) {
#pragma unroll
                for (int i = 0; i < 4; ++i) { v[i] = a0.v[0][i]; v[4 + i] = a1.v[0][i]; }
            } else if (!two_nb) {
#pragma unroll
                for (int i = 0; i < 4; ++i) { v[i] = a0.v[0][i]; v[4 + i] = 0.f; }
            } else {
#pragma unroll
                for (int i = 0; i < 4; ++i) { v[i] = d2.v[0][i]; v[4 + i] = d2.v[1][i]; }
            }
            const bool last = red_deposit(sh, red, r, w, lane, v, ok);
            if (!ok) break;
            if (last) {
                const float* rb0 = red + (r & 1) * NCW * 32 * 8;
                const int rg = 2 * tk.rb + rgl;
                if (tk.kind == 0) {
                    epilogue_a(p, rb0, slot, ncols, rg, lane);
                    if (rgl == 1) {
                        // both row-groups of the task are in h: publish
                        fence_proxy_async_global();
                        __threadfence();
                        __syncwarp();
                        if (lane == 0) atom_add_release_gpu(p.ctrl + MOE_CTRL_SLOT + slot, 1u);
                    }
                } else {
                    epilogue_b(p, S, rb0, slot, ncols, rg, lane);
                }
                red_release(sh, r, lane);
            }
            ++r;
        }
        if (!ok) break;
        if (tk.kind == 1) {
            __syncwarp();
            if (lane == 0) mbar_arrive(&sh.hfree[buf_h]);
            ++bseq;
        }
    }
    if (!ok) {
        set_error(p.ctrl, MOE_ERR_TIMEOUT);
        sh.abort_flag = 1;
    }
}

__global__ void __launch_bounds__(NTHREADS, 1) moe_decode_kernel(MoeParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* base = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t* ring = base;
    uint8_t* xh = ring + p.ns * MOE_STAGE_BYTES;
    float* red = (float*)(xh + p.xh_bytes);
    Shared& sh = *(Shared*)((uint8_t*)red + 2 * NCW * 32 * 8 * sizeof(float));
    const int hbytes_max = 4 * p.T * p.I;
    const int w = threadIdx.x >> 5;

    if (threadIdx.x == 0) {
        for (int s = 0; s < p.ns; ++s) {
            mbar_init(&sh.full[s], 1);
            mbar_init(&sh.empty[s], NCW);
        }
        for (int i = 0; i < QN; ++i) {
            mbar_init(&sh.tqf[i], 1);
            mbar_init(&sh.tqe[i], NCW);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sh.hfull[i], 1);
            mbar_init(&sh.hfree[i], NCW);
            sh.rcnt[i] = 0;
            sh.repoch[i] = i - 2;
        }
        mbar_init(&sh.xfree, NCW);
        sh.abort_flag = 0;
        sh.consumed = 0;
        fence_barrier_init();
    }
    if (w == NCW) {
        build_slots(p, sh.st);
    } else {
        // x (bf16 [T][H]) -> shared, fragment order [c][step][t][k 2t,2t+1,2t+8,2t+9]
        const int npairs = p.T * p.H / 2;
        const uint32_t* x32 = (const uint32_t*)p.x;
        for (int i = threadIdx.x; i < npairs; i += NCW * 32) {
            const int c = (2 * i) / p.H, k = (2 * i) % p.H;
            const int step = k >> 4, rr = k & 15;
            const int tt = (rr & 7) >> 1, half = rr >> 3;
            *(uint32_t*)(xh + c * p.x_stride + (step * 4 + tt) * 8 + half * 4) = x32[i];
        }
    }
    __syncthreads();
    if (w == NCW) {
        if ((threadIdx.x & 31) == 0) producer(p, sh, ring, xh, hbytes_max);
    } else {
        consumer(p, sh, ring, xh, hbytes_max, red);
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
size_t moe_decode_smem_bytes(int ns, int xh_bytes) {
    return 1024 + (size_t)ns * MOE_STAGE_BYTES + xh_bytes + 2 * NCW * 32 * 8 * sizeof(float) + sizeof(Shared);
}

cudaError_t moe_decode_launch(const MoeParams& p, int grid, cudaStream_t stream) {
    const size_t smem = moe_decode_smem_bytes(p.ns, p.xh_bytes);
    auto kern = moe_decode_kernel;
    // raise the dynamic shared-memory limit once (not a stream operation, so
    // it stays out of any graph capture after the first call)
    static int set_bytes[64] = {0};
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev < 64 && set_bytes[dev] < (int)smem) {
        err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (err != cudaSuccess) return err;
        set_bytes[dev] = (int)smem;
    }
    kern<<<grid, NTHREADS, smem, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace rfx
