// prefill.cu -- the MoE FFN for many tokens (prefill): the same mathematics
// as the decode path (m.mzlw.cn, "Lucebox专攻DeepSeek V4…", section "MoE 专家
// 并行": top-6 of 256 routed experts plus one shared expert, gate/up -> SwiGLU
// -> down, weighted combine) run as a grouped GEMM on the tcgen05 tensor
// cores.  The packed ROCmFPX-style blocks (taozi.news, "DeepSeek V4 Flash 在
// 128GB 锐龙 AI MAX+ 上跑到 32 tok/s", section "ROCmFPX：把 284B 权重压进
// 128 GB") are dequantised to bf16 in shared memory, once per (expert,
// 128-row tile, token tile), and fed to the tensor cores as the M = 128
// operand; the tokens routed to the expert are the N operand (16..256).
//
// Operand precision: every weight enters the MMA as bf16(level * scale)
// (rounded to nearest even from the exact product) and the SwiGLU output
// enters the down projection as bf16(h); accumulation is fp32 in tensor
// memory.
//
// Steps (one stream, six launches):
//   pf_count   tokens per routed expert in each slice of 1024 routed entries,
//              and the expert-id range check
//   pf_tiles   per-expert totals and first rows; token tiles of <= 256 rows:
//              the shared expert's first, then the routed experts by
//              descending token count (heaviest work first)
//   pf_place   rows grouped by expert, tokens in ascending order inside an
//              expert (stable, so the grouping is unique): token and weight
//   pf_gather  the routed rows of x copied into grouped order; y zeroed
//   pf_gemm<0> gate/up GEMM + SwiGLU -> h (bf16), per (tile, 128-row block of I)
//   pf_gemm<1> down GEMM, per (tile, 128-row block of H); the epilogue adds
//              w * d into y[token] (fp32 atomics: the order of the k + 1
//              additions per output element is not fixed)
#include <cuda.h>
#include <cuda_runtime.h>

#include "launch_util.h"
#include "moe_decode.h"
#include "prefill.h"
#include "rfx_layout.h"
#include "rfx_tile.cuh"
#include "tc.cuh"
#include "tmap.h"

namespace rfx {
namespace {

constexpr long long PF_WAIT = 1000000000LL;   // default SM clocks before a wait gives up (about half a second)

constexpr int W_PROD = 0;     // TMA loads of the token rows (B operand); hands out the units
constexpr int W_MMA = 1;      // tensor-memory allocation; first MMA issuer
constexpr int W_MMA2 = 2;     // second MMA issuer
constexpr int W_DQ0 = 3;      // dequantisation warps (count per mode below), then
constexpr int N_EPI = 4;      // 4 epilogue warps, one tensor-memory lane quarter each (warp % 4)
constexpr uint32_t TMEM_COLS = 512;
constexpr int CB_MAX = 128 * 17;   // bytes of the largest full chunk (FP4)
constexpr int PF_BOX_ROWS = 64;    // token rows per TMA box (the B stage holds 256)

// EX (exact precision): every dequantised weight is the bf16 pair hi + lo
// (hi = bf16(w), lo = bf16(w - hi): w = level * scale has at most 15
// significant bits, so the pair is exact), and the SwiGLU output is the bf16
// pair h1 + h2 (16 bits).  Gate/up: 2 MMAs per k-step and matrix; down: 4
// (hi h1, hi h2, lo h1, lo h2).  A stage holds the hi tiles of every matrix,
// then the lo tiles; MODE 1 stages hold the h1 rows, then the h2 rows.
template <int MODE, bool EX = false>
struct PfCfg {
    static constexpr int NMAT = MODE == 0 ? 2 : 1;                 // gate + up, or down
    static constexpr int NPART = EX ? 2 : 1;                        // weight tiles per matrix (hi, lo)
    static constexpr int BPART = (EX && MODE == 1) ? 2 : 1;         // token-row tiles per stage (h1, h2)
    // MODE 0: two dequantisation warps per 16-row group (gate, up); MODE 1: one
    static constexpr int N_DQ = MODE == 0 ? 16 : 8;
    static constexpr int W_EPI0 = W_DQ0 + N_DQ;
    static constexpr int THREADS = 32 * (W_EPI0 + N_EPI);
    static constexpr int UQ_READERS = 2 + N_DQ + N_EPI;           // MMA issuers, dequantisation and epilogue warps
    static constexpr int A_MAT = PF_BM * PF_BK * 2;                // 16 KB bf16 per matrix
    static constexpr int LO_OFF = NMAT * A_MAT;                     // the lo tiles after the hi tiles
    static constexpr int A_BYTES = NPART * NMAT * A_MAT;
    static constexpr int B_TILE = PF_TILE_N * PF_BK * 2;            // 32 KB bf16
    static constexpr int B_BYTES = BPART * B_TILE;
    static constexpr int NS = EX ? 2 : (MODE == 0 ? 3 : 4);         // stages of (dequantised A, token-row B)
    static constexpr int P_STAGE = N_DQ * CB_MAX;                   // one packed chunk per dequantisation warp
    static constexpr int NACC = MODE == 0 ? 1 : 2;                  // accumulator buffers of 256 (MODE 1) columns
    // MODE 0: issuer 0 runs the gate MMAs and issuer 1 the up MMAs of every
    // stage; MODE 1: issuer 0 the even and issuer 1 the odd stages
    static constexpr int EMPTY_ARRIVALS = MODE == 0 ? 2 : 1;
    // header (barriers) in the first 1 KB, then the rings from a 1024-byte boundary
    static constexpr size_t RINGS = (size_t)NS * (A_BYTES + B_BYTES) + (size_t)P_STAGE;
    static constexpr size_t SMEM = 1024 + RINGS;
    static_assert(A_MAT % 1024 == 0 && B_TILE % 1024 == 0, "swizzle atoms must stay 1024-byte aligned");
    static_assert(P_STAGE % 128 == 0, "bulk-copy destinations must stay 16-byte aligned");
    static_assert(SMEM <= 232448, "more shared memory than a B200 block may have");
};

constexpr int UQ = 4;                       // unit queue slots

struct PfShared {
    uint64_t full[4];     // stage ready: A written (one arrival per dequantisation warp) and B
                          // landed (1 arrival + bytes)
    uint64_t empty[4];    // stage read by the tensor cores (MMA commits)
    uint64_t first[2];    // MODE 1: the unit's first (zeroing) MMA has been issued
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint64_t uq_full[UQ];    // unit id published (producer)
    uint64_t uq_empty[UQ];   // unit id read by every other role
    uint64_t drain;
    volatile int uq[UQ];
    uint32_t tmem;
    volatile int abort;
    long long limit;   // SM clocks before a bounded wait gives up
};
static_assert(sizeof(PfShared) <= 1024, "barrier header must fit the first 1 KB");

__device__ __forceinline__ void pf_set_error(uint32_t* ctrl, uint32_t bits) { atomicOr(ctrl + PF_CTRL_ERR, bits); }

// Bounded wait; gives up when another role of the CTA has aborted or after
// sh.limit clocks (then records a timeout and aborts the CTA).
__device__ __noinline__ bool pf_wait(PfShared& sh, uint32_t* ctrl, uint64_t* bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (true) {
        if (mbar_try_wait_sleep(bar, parity, 20000u)) return true;
        if (sh.abort) return false;
        if (clock64() - t0 > sh.limit) {
            sh.abort = 1;
            pf_set_error(ctrl, MOE_ERR_TIMEOUT);
            return false;
        }
    }
}

// Bounded wait that does not give up on an abort: used before the CTA exits,
// so that no copy or MMA of this CTA is still writing its memory.
__device__ __noinline__ bool pf_wait_drain(uint32_t* ctrl, uint64_t* bar, uint32_t parity, long long limit) {
    const long long t0 = clock64();
    while (!mbar_try_wait_sleep(bar, parity, 20000u))
        if (clock64() - t0 > limit) {
            pf_set_error(ctrl, MOE_ERR_TIMEOUT);
            return false;
        }
    return true;
}

// Whole-warp wait: every lane acquires; the outcome is made uniform.
__device__ __forceinline__ bool pf_wait_warp(PfShared& sh, uint32_t* ctrl, uint64_t* bar, uint32_t parity) {
    const bool ok = pf_wait(sh, ctrl, bar, parity);
    return __all_sync(0xffffffffu, ok);
}

// ----------------------------------------------------------- grouping ---

// Routed entries t*k + j are cut into slices of PF_SLICE; a grouping CTA
// handles 8 experts (one warp each) of one slice.
__device__ __forceinline__ void grp_stage(const int32_t* __restrict__ src, int32_t* dst, int m) {
    for (int i = threadIdx.x; i < m; i += 256) dst[i] = src[i];
}

// cnt_part[slice][e]; the CTAs of expert block 0 also check every id against [0, E).
__global__ void __launch_bounds__(256) pf_count_kernel(const int32_t* __restrict__ idx, int n, int E,
                                                       int32_t* __restrict__ cnt_part, uint32_t* __restrict__ ctrl) {
    __shared__ __align__(16) int32_t s_idx[PF_SLICE];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int e = blockIdx.x * 8 + warp;
    const int base = blockIdx.y * PF_SLICE;
    const int m = min(PF_SLICE, n - base);
    grp_stage(idx + base, s_idx, m);
    __syncthreads();
    int c = 0;
    bool bad = false;
    for (int i0 = 0; i0 < m; i0 += 128) {
        const int i = i0 + 4 * lane;
        const int4 v = *reinterpret_cast<const int4*>(s_idx + i);
        const int vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < 4; ++j)
            if (i + j < m) {
                c += vv[j] == e;
                if (blockIdx.x == 0 && warp == 0) bad |= vv[j] < 0 || vv[j] >= E;
            }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
    if (lane == 0 && e < E) cnt_part[(long long)blockIdx.y * E + e] = c;
    if (__any_sync(0xffffffffu, bad) && lane == 0) pf_set_error(ctrl, MOE_ERR_EXPERT);
}

// The entries (t, j) routed to e take rows off[e] + (hits of e in the slices
// before this one) + ..., in ascending entry order t * k + j.  Per step a warp
// looks at 128 entries, lane L at entries 4L .. 4L+3: the hits of the lower
// lanes (4 ballots) plus the lane's own earlier hits give each hit its row.
__global__ void __launch_bounds__(256) pf_place_kernel(const int32_t* __restrict__ idx,
                                                       const float* __restrict__ wts, int n, int k, int E,
                                                       const int32_t* __restrict__ cnt_part,
                                                       const int32_t* __restrict__ off_e,
                                                       int32_t* __restrict__ perm_tok, float* __restrict__ perm_w) {
    __shared__ __align__(16) int32_t s_idx[PF_SLICE];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int e = blockIdx.x * 8 + warp;
    const int base = blockIdx.y * PF_SLICE;
    const int m = min(PF_SLICE, n - base);
    grp_stage(idx + base, s_idx, m);
    __syncthreads();
    if (e >= E) return;
    int off = 0;
    for (int s = lane; s < (int)blockIdx.y; s += 32) off += cnt_part[(long long)s * E + e];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) off += __shfl_xor_sync(0xffffffffu, off, o);
    off += off_e[e];
    const uint32_t lt = (1u << lane) - 1u;
    for (int i0 = 0; i0 < m; i0 += 128) {
        const int i = i0 + 4 * lane;
        const int4 v = *reinterpret_cast<const int4*>(s_idx + i);
        const bool h0 = i < m && v.x == e, h1 = i + 1 < m && v.y == e;
        const bool h2 = i + 2 < m && v.z == e, h3 = i + 3 < m && v.w == e;
        const uint32_t b0 = __ballot_sync(0xffffffffu, h0), b1 = __ballot_sync(0xffffffffu, h1);
        const uint32_t b2 = __ballot_sync(0xffffffffu, h2), b3 = __ballot_sync(0xffffffffu, h3);
        if (h0 | h1 | h2 | h3) {
            int pos = off + __popc(b0 & lt) + __popc(b1 & lt) + __popc(b2 & lt) + __popc(b3 & lt);
            const bool hv[4] = {h0, h1, h2, h3};
#pragma unroll
            for (int j = 0; j < 4; ++j)
                if (hv[j]) {
                    perm_tok[pos] = (base + i + j) / k;
                    perm_w[pos] = wts[base + i + j];
                    ++pos;
                }
        }
        off += __popc(b0) + __popc(b1) + __popc(b2) + __popc(b3);
    }
}

// Exclusive prefix sum over the 1024 threads of the block; *total gets the sum.
__device__ int block_excl_scan(int v, int* ws, int* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += u;
    }
    __syncthreads();
    if (lane == 31) ws[warp] = inc;
    __syncthreads();
    if (warp == 0) {
        const int s = ws[lane];
        int si = s;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int u = __shfl_up_sync(0xffffffffu, si, o);
            if (lane >= o) si += u;
        }
        ws[lane] = si - s;
        if (lane == 31) ws[32] = si;
    }
    __syncthreads();
    const int r = ws[warp] + inc - v;
    *total = ws[32];
    return r;
}

// One CTA of 1024 threads (E <= 1024): expert offsets, the descending-count
// order (ties: lower expert id first), and the token tiles.  A count c is cut
// into ceil(c / 256) tiles of nearly equal size.
__global__ void __launch_bounds__(1024) pf_tiles_kernel(PfParams p) {
    __shared__ int s_cnt[1024], s_off[1024], s_ord[1024];
    __shared__ int s_ws[33];
    const int tid = threadIdx.x;
    const int slices = (p.T * p.k + PF_SLICE - 1) / PF_SLICE;
    int c = 0;
    if (tid < p.E) {
        for (int s = 0; s < slices; ++s) c += p.cnt_part[(long long)s * p.E + tid];
        p.cnt[tid] = c;
    }
    s_cnt[tid] = c;
    int rows = 0;
    s_off[tid] = block_excl_scan(c, s_ws, &rows);
    if (tid < p.E) p.off[tid] = s_off[tid];
    __syncthreads();
    if (tid < p.E) {
        int r = 0;
        for (int e2 = 0; e2 < p.E; ++e2) {
            const int c2 = s_cnt[e2];
            r += c2 > c || (c2 == c && e2 < tid);
        }
        s_ord[r] = tid;
    }
    __syncthreads();
    const int eo = tid < p.E ? s_ord[tid] : -1;
    const int co = eo >= 0 ? s_cnt[eo] : 0;
    const int nt = (co + PF_TILE_N - 1) / PF_TILE_N;
    int nt_total = 0;
    const int tb = block_excl_scan(nt, s_ws, &nt_total);
    const int nts = p.has_shared ? (p.T + PF_TILE_N - 1) / PF_TILE_N : 0;
    if (nt > 0) {
        const int sz = (co + nt - 1) / nt;
        for (int j = 0; j < nt; ++j)
            p.tiles[nts + tb + j] = make_int4(s_off[eo] + j * sz, min(sz, co - j * sz), eo, 0);
    }
    if (tid < nts) {
        const int sz = (p.T + nts - 1) / nts;
        p.tiles[tid] = make_int4(p.T * p.k + tid * sz, min(sz, p.T - tid * sz), -1, 0);
    }
    if (tid == 0) {
        p.ctrl[PF_CTRL_NTILES] = (uint32_t)(nts + nt_total);
        p.ctrl[PF_CTRL_ROWS] = (uint32_t)rows;
        p.ctrl[PF_CTRL_NEXT0] = 0;
        p.ctrl[PF_CTRL_NEXT1] = 0;
    }
}

// x rows in grouped order (16-byte copies), and y = 0.
__global__ void __launch_bounds__(256) pf_gather_kernel(PfParams p) {
    const int nch = p.H / 8;   // 16-byte chunks per row
    const long long rows = (long long)p.ctrl[PF_CTRL_ROWS];
    const long long items = rows * nch;
    const long long stride = (long long)gridDim.x * blockDim.x;
    const uint4* xs = reinterpret_cast<const uint4*>(p.x);
    uint4* xd = reinterpret_cast<uint4*>(p.xp);
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < items; i += stride) {
        const long long r = i / nch;
        const int ch = (int)(i - r * nch);
        xd[i] = __ldg(xs + (long long)p.perm_tok[r] * nch + ch);
    }
    float4* y4 = reinterpret_cast<float4*>(p.y);
    const long long ny = (long long)p.T * p.H / 4;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < ny; i += stride)
        y4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
}

// --------------------------------------------------------- grouped GEMM ---

struct PfUnit {
    int row0, n, e, rt, npad;
};

__device__ __forceinline__ PfUnit pf_unit(const PfParams& p, int u, int RT) {
    const int4 t = p.tiles[u / RT];
    PfUnit U;
    U.row0 = t.x;
    U.n = t.y;
    U.e = t.z;
    U.rt = u % RT;
    U.npad = (t.y + 15) & ~15;
    return U;
}

// One lane's share of a full chunk (8 tiles = 16 rows x 256 k) of one matrix,
// read from the packed stage in shared memory (slab-major layout,
// include/rfx.h: every 128-bit load of the warp reads 512 contiguous bytes).
template <int F>
struct PfChunk {
    static constexpr int NW = 4 * F;
    static constexpr int NSW = F == 4 ? 4 : 8;
    uint32_t wd[NW];
    uint32_t sc[NSW];
    __device__ __forceinline__ void load(const uint8_t* ch, int lane, int g) {
#pragma unroll
        for (int i = 0; i < F; ++i) {
            const uint4 v = lds128(ch + (i * 32 + lane) * 16);
            wd[4 * i] = v.x; wd[4 * i + 1] = v.y; wd[4 * i + 2] = v.z; wd[4 * i + 3] = v.w;
        }
        constexpr int CODE = Plane<F>::CODE_BYTES;
#pragma unroll
        for (int i = 0; i < NSW / 4; ++i) {
            const uint4 v = lds128(ch + CODE + (i * 8 + g) * 16);
            sc[4 * i] = v.x; sc[4 * i + 1] = v.y; sc[4 * i + 2] = v.z; sc[4 * i + 3] = v.w;
        }
    }
};

// Tile B of a chunk -> bf16 into the swizzled A tile.  Register r of the lane
// holds row g + 8 (r & 1), k = 32 (B & 1) + 16 (r >> 2) + 8 ((r >> 1) & 1) + 2t
// (+1 in the high half) of the 64-wide stage; its 4 bytes go to 16-byte chunk
// k / 8 of that row, stored at chunk position (k / 8) ^ g.  `base` is the
// stage's matrix tile address plus the lane's row-group, g and t offsets; xo[c]
// = ((c ^ g) << 4).
template <int F, int B, int LO>
__device__ __forceinline__ void pf_decode_tile(const PfChunk<F>& c, const uint32_t* sh, uint32_t base,
                                               const uint32_t* xo) {
    uint32_t a[8];
    plane_regs<F, B>(c.wd, sh, a);
    constexpr int S = Plane<F>::s_of(B);
    constexpr uint32_t MAGIC = ((uint32_t)(25 - S) << 10) * 0x10001u;   // fp16 2^(10-S) in both halves
    constexpr float K = -((float)(1 << (10 - S)) + Plane<F>::OFF);
    constexpr int BP = B & 1;
    if constexpr (F == 4) {
        const uint32_t w = c.sc[B >> 1] >> (16 * (B & 1));
        const float s0 = scale_e8m0(w & 0xFFu), s1 = scale_e8m0((w >> 8) & 0xFFu);
#pragma unroll
        for (int r = 0; r < 8; ++r) {
            const int cidx = 4 * BP + 2 * (r >> 2) + ((r >> 1) & 1);
            if constexpr (LO > 0) {
                uint32_t hi, lo;
                deq_pair_pow2scale_hilo(a[r] | MAGIC, K, (r & 1) ? s1 : s0, hi, lo);
                sts32(base + (r & 1) * 1024 + xo[cidx], hi);
                sts32(base + LO + (r & 1) * 1024 + xo[cidx], lo);
            } else {
                sts32(base + (r & 1) * 1024 + xo[cidx], deq_pair_pow2scale(a[r] | MAGIC, K, (r & 1) ? s1 : s0));
            }
        }
    } else {
        const uint32_t w = c.sc[B];
        const float2 s = scale_f16x2(w);
        const float C0 = K * s.x, C1 = K * s.y;
#pragma unroll
        for (int r = 0; r < 8; ++r) {
            const uint32_t v = a[r] | MAGIC;
            const int cidx = 4 * BP + 2 * (r >> 2) + ((r >> 1) & 1);
            if constexpr (LO > 0) {
                uint32_t hi, lo;
                if (r & 1) deq_pair_f16scale_hilo<1>(v, w, C1, hi, lo);
                else deq_pair_f16scale_hilo<0>(v, w, C0, hi, lo);
                sts32(base + (r & 1) * 1024 + xo[cidx], hi);
                sts32(base + LO + (r & 1) * 1024 + xo[cidx], lo);
            } else {
                const uint32_t out = (r & 1) ? deq_pair_f16scale<1>(v, w, C1) : deq_pair_f16scale<0>(v, w, C0);
                sts32(base + (r & 1) * 1024 + xo[cidx], out);
            }
        }
    }
}

template <int F, int KK, int LO>
__device__ __forceinline__ void pf_decode_kstep(const PfChunk<F>& c, const uint32_t* sh, uint32_t base,
                                                const uint32_t* xo) {
    pf_decode_tile<F, 2 * KK, LO>(c, sh, base, xo);
    pf_decode_tile<F, 2 * KK + 1, LO>(c, sh, base, xo);
}

template <int F>
__device__ __forceinline__ void pf_shift(const PfChunk<F>& c, uint32_t* sh) {
    constexpr int SH = F == 2 ? 10 : (F == 3 ? 9 : 8);
#pragma unroll
    for (int i = 0; i < 4 * F; ++i) sh[i] = c.wd[i] >> SH;
}

struct PfRings {
    uint8_t* a;         // NS x dequantised A tiles (gate, up / down)
    uint8_t* b;         // NS x token-row B tiles
    uint8_t* pk;        // per dequantisation warp: its packed chunk [CB_MAX]
};

// Where the packed chunks of (unit, 256-wide k block) of one warp's row-group
// and matrix come from.
struct PfSrc {
    const uint8_t* m;   // the row-group's stream
    int cb;             // chunk bytes
    int f;
};

// rg = 16-row group of the unit's 128-row block, sub = the warp's half (MODE 0:
// gate or up matrix; MODE 1: even or odd tiles of the down matrix)
__device__ __forceinline__ PfSrc pf_src(const PfParams& p, int mode, const PfUnit& U, int rg, int sub) {
    PfSrc S;
    S.f = mode == 0 ? (U.e >= 0 ? p.fA : p.fsA) : (U.e >= 0 ? p.fB : p.fsB);
    long long og = (long long)U.e * p.sg, ou = (long long)U.e * p.su, od = (long long)U.e * p.sd;
    if (p.mix && U.e >= 0) {   // ROCmFPX MIX: the expert's own format and place
        const MoeMixEntry* m = p.mix + U.e;
        S.f = mode == 0 ? __ldg(&m->fa) : __ldg(&m->fb);
        og = __ldg(&m->og); ou = __ldg(&m->ou); od = __ldg(&m->od);
    }
    const int K = mode == 0 ? p.H : p.I;
    const long long rgb = (long long)(K / 32) * 16 * rfx_block_bytes(S.f);
    S.cb = 128 * rfx_block_bytes(S.f);
    const long long off = ((long long)U.rt * (PF_BM / 16) + rg) * rgb;
    if (mode == 0)
        S.m = (sub == 0 ? (U.e >= 0 ? p.gate + og : p.shg) : (U.e >= 0 ? p.up + ou : p.shu)) + off;
    else
        S.m = (U.e >= 0 ? p.down + od : p.shd) + off;
    return S;
}

// The warp copies chunk `ch` into its slot with 16-byte asynchronous copies,
// one commit group per lane.
__device__ __forceinline__ void pf_prefetch(const PfSrc& S, int ch, uint32_t slot, int lane, uint64_t pol) {
    const int pieces = S.cb / 16;
    const uint8_t* src = S.m + (long long)ch * S.cb;
    for (int i = lane; i < pieces; i += 32) cp_async16(slot + 16 * i, src + 16 * i, pol);
    cp_async_commit();
}

// One 256-wide k block of one unit by one warp: the packed chunk from the
// warp's slot into registers, the next copy started into the freed slot, then
// its part of 4 stages of A written (MODE 0: both tiles of its matrix per
// stage; MODE 1: the tile of its parity).  `base` already points at the
// warp's matrix and row-group.  Returns false on abort.
template <int MODE, bool EX, int F>
__device__ bool pf_dq_chunk(const PfParams& p, PfShared& sh, const PfRings& R, const uint8_t* slot, int lane, int g,
                            int sub, const uint32_t* xo, uint32_t lane_off, int& gstep, const PfSrc* nsrc, int nch,
                            uint32_t slot_s, uint64_t pol) {
    using Cfg = PfCfg<MODE, EX>;
    constexpr int LO = EX ? Cfg::LO_OFF : 0;
    cp_async_wait_all();
    __syncwarp();
    PfChunk<F> c0;
    c0.load(slot, lane, g);
    __syncwarp();
    if (nsrc) pf_prefetch(*nsrc, nch, slot_s, lane, pol);
    uint32_t s0[4 * F];
    pf_shift<F>(c0, s0);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
        const int s = gstep % Cfg::NS;
        const uint32_t ph = (uint32_t)(gstep / Cfg::NS) & 1u;
        if (!pf_wait_warp(sh, p.ctrl, &sh.empty[s], ph ^ 1u)) return false;
        const uint32_t base = smem_u32(R.a + (size_t)s * Cfg::A_BYTES) + lane_off;
        if (MODE == 0 || Cfg::N_DQ == 8) {   // both tiles of the stage
            switch (kk) {
                case 0: pf_decode_kstep<F, 0, LO>(c0, s0, base, xo); break;
                case 1: pf_decode_kstep<F, 1, LO>(c0, s0, base, xo); break;
                case 2: pf_decode_kstep<F, 2, LO>(c0, s0, base, xo); break;
                default: pf_decode_kstep<F, 3, LO>(c0, s0, base, xo); break;
            }
        } else if (sub == 0) {
            switch (kk) {
                case 0: pf_decode_tile<F, 0, LO>(c0, s0, base, xo); break;
                case 1: pf_decode_tile<F, 2, LO>(c0, s0, base, xo); break;
                case 2: pf_decode_tile<F, 4, LO>(c0, s0, base, xo); break;
                default: pf_decode_tile<F, 6, LO>(c0, s0, base, xo); break;
            }
        } else {
            switch (kk) {
                case 0: pf_decode_tile<F, 1, LO>(c0, s0, base, xo); break;
                case 1: pf_decode_tile<F, 3, LO>(c0, s0, base, xo); break;
                case 2: pf_decode_tile<F, 5, LO>(c0, s0, base, xo); break;
                default: pf_decode_tile<F, 7, LO>(c0, s0, base, xo); break;
            }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh.full[s]);
        ++gstep;
    }
    return true;
}

// silu(g) * u with the hardware exponential and a fast reciprocal (relative
// error a few fp32 ulps, far below the bf16 rounding that follows); the far
// negative tail separately, so that tiny h keep their value.
__device__ __forceinline__ float silu_mul(float g, float u) {
    return g >= -64.f ? __fdividef(g, 1.0f + __expf(-g)) * u : silu_mul_tail(g, u);
}

__device__ __forceinline__ uint16_t f32_to_bf16_rne(float v) {
    uint16_t r;
    asm("cvt.rn.bf16.f32 %0, %1;" : "=h"(r) : "f"(v));
    return r;
}

// Unit i of this CTA from the queue (whole warp or a single thread); -1 ends.
__device__ __forceinline__ int pf_take_unit(PfShared& sh, uint32_t* ctrl, int i, bool warp_wide, bool& ok) {
    const int slot = i % UQ;
    const uint32_t ph = (uint32_t)(i / UQ) & 1u;
    ok = warp_wide ? pf_wait_warp(sh, ctrl, &sh.uq_full[slot], ph) : pf_wait(sh, ctrl, &sh.uq_full[slot], ph);
    if (!ok) return -1;
    const int u = sh.uq[slot];
    if (warp_wide) __syncwarp();
    if (!warp_wide || (threadIdx.x & 31) == 0) mbar_arrive(&sh.uq_empty[slot]);
    return u;
}

// Persistent grouped GEMM, one CTA per SM.  Units (token tile, 128-row block)
// are taken from a global counter in the tiles' order (heaviest first) by the
// producer thread and passed to the other roles through a small queue.
// MODE 0: gate/up + SwiGLU -> hp.  MODE 1: down, y[token] += w * d.
template <int MODE, bool EX>
__global__ void __launch_bounds__(PfCfg<MODE, EX>::THREADS, 1)
    pf_gemm_kernel(const PfParams p, const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmX) {
    using Cfg = PfCfg<MODE, EX>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    PfShared& sh = *reinterpret_cast<PfShared*>(smem_raw);
    // rings from the first 1024-byte boundary after the header; the launch
    // reserves 1 KB for the header, so the block's dynamic shared memory must
    // start 1024-byte aligned (checked below)
    const uint32_t off = ((smem_u32(smem_raw) + (uint32_t)sizeof(PfShared) + 1023u) & ~1023u) - smem_u32(smem_raw);
    PfRings R;
    R.a = smem_raw + off;
    R.b = R.a + (size_t)Cfg::NS * Cfg::A_BYTES;
    R.pk = R.b + (size_t)Cfg::NS * Cfg::B_BYTES;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (off > 1024u) {   // the rings would overrun the allocation: report and do nothing
        if (threadIdx.x == 0) pf_set_error(p.ctrl, MOE_ERR_TIMEOUT);
        return;
    }

    if (threadIdx.x == 0) {
        for (int s = 0; s < Cfg::NS; ++s) {
            mbar_init(&sh.full[s], Cfg::N_DQ + 1);
            mbar_init(&sh.empty[s], Cfg::EMPTY_ARRIVALS);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sh.acc_full[b], 2);
            mbar_init(&sh.acc_empty[b], N_EPI);
            mbar_init(&sh.first[b], 1);
        }
        for (int q = 0; q < UQ; ++q) {
            mbar_init(&sh.uq_full[q], 1);
            mbar_init(&sh.uq_empty[q], Cfg::UQ_READERS);
        }
        mbar_init(&sh.drain, 2);
        sh.abort = 0;
        sh.limit = p.wait_limit;
        fence_barrier_init();
    }
    if (warp == W_MMA) {
        __syncwarp();
        tmem_alloc(&sh.tmem, TMEM_COLS);
        tmem_relinquish();
    }
    if (warp == W_PROD && lane == 0) {
        tma_prefetch_desc(&tmB);
        if (MODE == 0) tma_prefetch_desc(&tmX);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sh.tmem;

    const int RT = (MODE == 0 ? p.I : p.H) / PF_BM;
    const int K = MODE == 0 ? p.H : p.I;
    const int nk = K / PF_BK;
    const int nunits = (int)p.ctrl[PF_CTRL_NTILES] * RT;
    const int rk = p.T * p.k;

    if (warp == W_PROD) {
        if (lane == 0) {
            const uint64_t pol = policy_evict_last();
            uint32_t* next = p.ctrl + (MODE == 0 ? PF_CTRL_NEXT0 : PF_CTRL_NEXT1);
            // units are published one ahead of the one being loaded, so that the
            // dequantisation warps can start fetching the next unit's weights
            // while the current one is still in flight
            auto publish = [&](int i, int u) -> bool {
                const int slot = i % UQ;
                if (!pf_wait(sh, p.ctrl, &sh.uq_empty[slot], ((uint32_t)(i / UQ) & 1u) ^ 1u)) return false;
                sh.uq[slot] = u;
                mbar_arrive(&sh.uq_full[slot]);
                return true;
            };
            auto grab = [&]() -> int {
                const int u = (int)atomicAdd(next, 1u);
                return u < nunits ? u : -1;
            };
            int gstep = 0;
            bool ok = true;
            // tests of the error path only: wait for the release of a stage that
            // nothing has loaded (it never comes; the wait times out)
            if (MODE == 1 && p.fault == 3) ok = pf_wait(sh, p.ctrl, &sh.empty[0], 0u);
            int u = ok ? grab() : -1;
            ok = ok && publish(0, u);
            for (int i = 0; ok && u >= 0; ++i) {
                const int un = grab();
                if (!publish(i + 1, un)) break;
                const PfUnit U = pf_unit(p, u, RT);
                const bool shx = MODE == 0 && U.e < 0;
                const void* tm = shx ? (const void*)&tmX : (const void*)&tmB;
                const int rbase = shx ? U.row0 - rk : U.row0;
                const int nbox = (U.npad + PF_BOX_ROWS - 1) / PF_BOX_ROWS;
                for (int ks = 0; ks < nk; ++ks, ++gstep) {
                    const int s = gstep % Cfg::NS;
                    const uint32_t ph = (uint32_t)(gstep / Cfg::NS) & 1u;
                    if (!pf_wait(sh, p.ctrl, &sh.empty[s], ph ^ 1u)) { ok = false; break; }
                    mbar_arrive_expect_tx(&sh.full[s], (uint32_t)(Cfg::BPART * nbox) * (PF_BOX_ROWS * PF_BK * 2));
                    uint8_t* dst = R.b + (size_t)s * Cfg::B_BYTES;
                    // exact down: the h1 rows, then the h2 rows (hrows further in the same map)
                    for (int part = 0; part < Cfg::BPART; ++part)
                        for (int j = 0; j < nbox; ++j)
                            tma_load_2d(dst + part * Cfg::B_TILE + j * (PF_BOX_ROWS * PF_BK * 2), tm, ks * PF_BK,
                                        rbase + part * (rk + p.T) + PF_BOX_ROWS * j, &sh.full[s], pol);
                }
                u = un;
            }
            // no copy may still be landing when the CTA exits: the last stages
            // this thread filled must have completed (or the CTA aborted, and
            // then the bounded wait gives up)
            for (int i = 1; i <= Cfg::NS && gstep - i >= 0; ++i) {
                const int gi = gstep - i;
                (void)pf_wait_drain(p.ctrl, &sh.full[gi % Cfg::NS], (uint32_t)(gi / Cfg::NS) & 1u, sh.limit);
            }
        }
    } else if (warp == W_MMA || warp == W_MMA2) {
        if (lane == 0) {
            const int who = warp - W_MMA;
            int gstep = 0;
            for (int i = 0;; ++i) {
                bool ok;
                const int u = pf_take_unit(sh, p.ctrl, i, false, ok);
                if (u < 0) break;
                const PfUnit U = pf_unit(p, u, RT);
                const uint32_t idesc = idesc_bf16_m128((uint32_t)U.npad);
                const int b = i % Cfg::NACC, use = i / Cfg::NACC;
                if (!pf_wait(sh, p.ctrl, &sh.acc_empty[b], (uint32_t)(use & 1) ^ 1u)) break;
                tc_fence_after();
                // MODE 0: this issuer's own accumulator (gate or up); MODE 1: the
                // unit's buffer, shared by both issuers
                const uint32_t dacc = tmem + (uint32_t)((MODE == 0 ? who : b) * 256);
                const uint32_t aoff = MODE == 0 ? (uint32_t)(who * Cfg::A_MAT) : 0u;
                for (int ks = 0; ks < nk; ++ks, ++gstep) {
                    if (MODE == 1 && (ks & 1) != who) continue;
                    const int s = gstep % Cfg::NS;
                    if (!pf_wait(sh, p.ctrl, &sh.full[s], (uint32_t)(gstep / Cfg::NS) & 1u)) {
                        ok = false;
                        break;
                    }
                    if (MODE == 1 && who == 1 && ks == 1 &&
                        !pf_wait(sh, p.ctrl, &sh.first[b], (uint32_t)(use & 1))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t aaddr = smem_u32(R.a + (size_t)s * Cfg::A_BYTES) + aoff;
                    const uint32_t baddr = smem_u32(R.b + (size_t)s * Cfg::B_BYTES);
#pragma unroll
                    for (int kk = 0; kk < PF_BK / 16; ++kk) {
                        tc_mma_bf16(dacc, sw128_desc(aaddr + kk * 32), sw128_desc(baddr + kk * 32), idesc,
                                    (ks | kk) != 0);
                        if constexpr (EX) {   // the remaining products of the hi/lo pairs, in a fixed order
                            const uint32_t alo = aaddr + Cfg::LO_OFF + kk * 32;
                            if constexpr (MODE == 1) {
                                const uint32_t b2 = baddr + Cfg::B_TILE + kk * 32;
                                tc_mma_bf16(dacc, sw128_desc(aaddr + kk * 32), sw128_desc(b2), idesc, true);
                                tc_mma_bf16(dacc, sw128_desc(alo), sw128_desc(baddr + kk * 32), idesc, true);
                                tc_mma_bf16(dacc, sw128_desc(alo), sw128_desc(b2), idesc, true);
                            } else {
                                tc_mma_bf16(dacc, sw128_desc(alo), sw128_desc(baddr + kk * 32), idesc, true);
                            }
                        }
                    }
                    tc_commit(&sh.empty[s]);
                    // the zeroing MMA is issued: the other issuer may add to the buffer
                    if (MODE == 1 && ks == 0) {
                        tc_fence_before();
                        mbar_arrive(&sh.first[b]);
                    }
                }
                if (!ok) break;
                tc_commit(&sh.acc_full[b]);
            }
            tc_commit(&sh.drain);
            (void)pf_wait_drain(p.ctrl, &sh.drain, 0, sh.limit);
        }
    } else if (warp < Cfg::W_EPI0) {
        const int d = warp - W_DQ0;
        const int rg = Cfg::N_DQ == 16 ? d >> 1 : d, sub = Cfg::N_DQ == 16 ? d & 1 : 0;
        const int g = lane >> 2, t = lane & 3;
        uint32_t xo[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) xo[c] = (uint32_t)((c ^ g) << 4);
        // the warp's matrix (MODE 0) and row-group inside the stage's A tiles
        const uint32_t lane_off = (uint32_t)((MODE == 0 ? sub * Cfg::A_MAT : 0) + 2 * rg * 1024 + g * 128 + 4 * t);
        const uint8_t* slot = R.pk + (size_t)d * CB_MAX;
        const uint32_t slot_s = smem_u32(slot);
        const uint64_t pol = policy_evict_first();
        const int nch = nk / 4;
        int gstep = 0;
        bool ok;
        int u = pf_take_unit(sh, p.ctrl, 0, true, ok);
        PfSrc cur{};
        if (u >= 0) {
            cur = pf_src(p, MODE, pf_unit(p, u, RT), rg, sub);
            pf_prefetch(cur, 0, slot_s, lane, pol);
        }
        for (int i = 0; u >= 0; ++i) {
            int un = -1;
            PfSrc nxt{};
            for (int ch = 0; ch < nch && ok; ++ch) {
                const PfSrc* ns = nullptr;
                int nc = 0;
                if (ch + 1 < nch) {
                    ns = &cur;
                    nc = ch + 1;
                } else {
                    un = pf_take_unit(sh, p.ctrl, i + 1, true, ok);
                    if (!ok) break;
                    if (un >= 0) {
                        nxt = pf_src(p, MODE, pf_unit(p, un, RT), rg, sub);
                        ns = &nxt;
                    }
                }
                if (cur.f == 2) ok = pf_dq_chunk<MODE, EX, 2>(p, sh, R, slot, lane, g, sub, xo, lane_off, gstep, ns, nc, slot_s, pol);
                else if (cur.f == 3) ok = pf_dq_chunk<MODE, EX, 3>(p, sh, R, slot, lane, g, sub, xo, lane_off, gstep, ns, nc, slot_s, pol);
                else ok = pf_dq_chunk<MODE, EX, 4>(p, sh, R, slot, lane, g, sub, xo, lane_off, gstep, ns, nc, slot_s, pol);
            }
            if (!ok) break;
            u = un;
            cur = nxt;
        }
        cp_async_wait_all();   // nothing may still be landing in the slot when the CTA exits
    } else {
        const int q = warp & 3;   // tensor-memory lane quarter this warp may read
        const uint32_t tq = tmem + ((uint32_t)(32 * q) << 16);
        for (int i = 0;; ++i) {
            bool ok;
            const int u = pf_take_unit(sh, p.ctrl, i, true, ok);
            if (u < 0) break;
            const PfUnit U = pf_unit(p, u, RT);
            const int b = i % Cfg::NACC, use = i / Cfg::NACC;
            if (!pf_wait_warp(sh, p.ctrl, &sh.acc_full[b], (uint32_t)use & 1u)) break;
            tc_fence_after();
            const int row = U.rt * PF_BM + 32 * q + lane;
            if (MODE == 0) {
                uint16_t* hrow = p.hp + row;
                for (int c0 = 0; c0 < U.n; c0 += 16) {
                    uint32_t gv[16], uv[16];
                    tmem_ld16(tq + (uint32_t)c0, gv);
                    tmem_ld16(tq + 256u + (uint32_t)c0, uv);
                    tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 16; ++j)
                        if (c0 + j < U.n) {
                            const float hv = silu_mul(__uint_as_float(gv[j]), __uint_as_float(uv[j]));
                            const uint16_t h1 = f32_to_bf16_rne(hv);
                            hrow[(long long)(U.row0 + c0 + j) * p.I] = h1;
                            if constexpr (EX)   // h2 = bf16(h - h1): h1 + h2 carries 16 bits of h
                                hrow[((long long)(rk + p.T) + U.row0 + c0 + j) * p.I] =
                                    f32_to_bf16_rne(hv - __uint_as_float((uint32_t)h1 << 16));
                        }
                }
            } else {
                float* ycol = p.y + row;
                const uint32_t tb = tq + (uint32_t)(b * 256);
                for (int c0 = 0; c0 < U.n; c0 += 32) {
                    int tok = 0;
                    float wv = 0.f;
                    if (c0 + lane < U.n) {
                        const int pr = U.row0 + c0 + lane;
                        tok = U.e >= 0 ? p.perm_tok[pr] : pr - rk;
                        wv = U.e >= 0 ? p.perm_w[pr] : 1.0f;
                    }
#pragma unroll
                    for (int hf = 0; hf < 2; ++hf) {
                        if (c0 + 16 * hf >= U.n) break;
                        uint32_t dv[16];
                        tmem_ld16(tb + (uint32_t)(c0 + 16 * hf), dv);
                        tmem_ld_wait();
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const int c = c0 + 16 * hf + j;
                            const int tk = __shfl_sync(0xffffffffu, tok, 16 * hf + j);
                            const float ww = __shfl_sync(0xffffffffu, wv, 16 * hf + j);
                            if (c < U.n) atomicAdd(ycol + (long long)tk * p.H, ww * __uint_as_float(dv[j]));
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sh.acc_empty[b]);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == W_MMA) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

// ------------------------------------------------------------- host side ---

// bf16 matrix [rows][cols], boxes of PF_BK columns x PF_BOX_ROWS rows.
bool make_tmap(CUtensorMap* m, const void* base, long long rows, long long cols) {
    static_assert(PF_BK == 64, "the tensor maps' boxes are 64 columns wide");
    return make_tmap_bf16(m, base, rows, cols, PF_BOX_ROWS);
}

}  // namespace

size_t pf_gemm_smem_bytes(int mode, bool exact) {
    if (exact) return mode == 0 ? PfCfg<0, true>::SMEM : PfCfg<1, true>::SMEM;
    return mode == 0 ? PfCfg<0>::SMEM : PfCfg<1>::SMEM;
}

long long pf_default_wait_limit() { return PF_WAIT; }

template <bool EX>
static cudaError_t pf_gemm_limits() {
    static SmemLimit limit[2];
    cudaError_t e = limit[0].ensure((const void*)pf_gemm_kernel<0, EX>, (int)pf_gemm_smem_bytes(0, EX));
    if (e != cudaSuccess) return e;
    return limit[1].ensure((const void*)pf_gemm_kernel<1, EX>, (int)pf_gemm_smem_bytes(1, EX));
}

cudaError_t pf_launch(const PfParams& p, int sms, cudaStream_t stream) {
    cudaError_t e = p.exact ? pf_gemm_limits<true>() : pf_gemm_limits<false>();
    if (e != cudaSuccess) return e;
    CUtensorMap tm_xp, tm_x, tm_h;
    const long long rk = (long long)p.T * p.k;
    // the h rows (exact: h1 rows, then as many h2 rows)
    if (!make_tmap(&tm_xp, p.xp, rk, p.H) || !make_tmap(&tm_x, p.x, p.T, p.H) ||
        !make_tmap(&tm_h, p.hp, (p.exact ? 2 : 1) * (rk + p.T), p.I))
        return cudaErrorInvalidValue;
    const int n = p.T * p.k;
    const dim3 gg((p.E + 7) / 8, (n + PF_SLICE - 1) / PF_SLICE);
    (void)cudaGetLastError();   // an earlier call's launch error is not this call's
    pf_count_kernel<<<gg, 256, 0, stream>>>(p.idx, n, p.E, p.cnt_part, p.ctrl);
    pf_tiles_kernel<<<1, 1024, 0, stream>>>(p);
    pf_place_kernel<<<gg, 256, 0, stream>>>(p.idx, p.wts, n, p.k, p.E, p.cnt_part, p.off, p.perm_tok, p.perm_w);
    pf_gather_kernel<<<sms * 4, 256, 0, stream>>>(p);
    if (p.exact) {
        pf_gemm_kernel<0, true><<<sms, PfCfg<0, true>::THREADS, pf_gemm_smem_bytes(0, true), stream>>>(p, tm_xp, tm_x);
        pf_gemm_kernel<1, true><<<sms, PfCfg<1, true>::THREADS, pf_gemm_smem_bytes(1, true), stream>>>(p, tm_h, tm_h);
    } else {
        pf_gemm_kernel<0, false><<<sms, PfCfg<0>::THREADS, pf_gemm_smem_bytes(0, false), stream>>>(p, tm_xp, tm_x);
        pf_gemm_kernel<1, false><<<sms, PfCfg<1>::THREADS, pf_gemm_smem_bytes(1, false), stream>>>(p, tm_h, tm_h);
    }
    return cudaGetLastError();
}

}  // namespace rfx
