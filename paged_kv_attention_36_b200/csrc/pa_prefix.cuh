// pa_prefix.cuh -- shared-prefix ("cascade") attention for decode.
//
// With prefix caching, sequences that start with the same tokens hold the
// same physical blocks at the start of their block tables.  A group is a
// run of consecutive sequences [off[i], off[i+1]) whose first P_i table
// entries are those shared blocks.  Decode over the group would stream the
// P_i shared pages once per member; here the queries of all members attend
// to them once instead.  For kv head g the rows are (member m, query head
// g*G + j), so a tile of rows against a page of 16 prefix tokens is a dense
// [rows x 16] x [16 x D] contraction, done on the tensor cores (mma.sync
// m16n8k16, bf16 in, fp32 accumulate).  The prefix pages are split into
// `splits` ranges over blockIdx.z; each (range, member, head) leaves an fp32
// split-KV partial (normalised output, max logit in base 2, exp-sum) that
// the decode kernel folds into the member's own pages by log-sum-exp.
//
// CTA = (group, row tile, kv head, key range).  Consumer warp w owns rows
// 16w .. 16w+15 of the tile; warp NW streams the range's pages (K and V
// tiles of the group's first member's blocks, one tiled TMA copy each, in
// the 128-byte-swizzled panel layout of the decode) into a ring of RS
// stages that every consumer warp reads (a stage is free when all have
// arrived).
//
// Per page and warp (FlashAttention-2 fragment flow): S[16 x 16] = Q . K^T
// with K rows from ldmatrix; each row's max over the 4 lanes that hold it;
// P = exp2(S - m) packed from the accumulator fragments straight into the A
// operand of O[16 x D] += P . V (V rows from ldmatrix.trans).  P is split
// into a bf16 high part and a bf16 remainder, both multiplied, as in the
// decode.
#pragma once

#include "pa_device.cuh"

namespace pa {

// Sixteen query rows of one warp against staged (block, kv head) tiles of 16
// tokens (128-byte-swizzled panels, see tile_off), FlashAttention-2
// fragment flow on mma.sync m16n8k16 (bf16 in, fp32 accumulate).  Lane l
// holds rows lr = l/4 and lr+8 of the 16: its query fragments, and the
// accumulator columns 8*nt + 2*(l%4), +1 of both rows.
template <int D>
struct RowTile {
    static constexpr int KS = D / 16;
    uint32_t qa[KS][4];
    float o[D / 8][4];
    float m0, m1, l0, l1;  // rows lr and lr + 8: running max (base 2), running sum

    // row0 / row1: the D bf16 query values of rows lr and lr+8, or nullptr (zeros)
    __device__ __forceinline__ void load_q(const uint8_t* row0, const uint8_t* row1, int lane) {
        const int lc = (lane & 3) * 2;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const uint32_t* row = reinterpret_cast<const uint32_t*>(e ? row1 : row0);
#pragma unroll
            for (int ks = 0; ks < KS; ++ks) {
                qa[ks][e] = row ? __ldg(row + (16 * ks + lc) / 2) : 0u;          // a0a1 / a2a3: columns lc, lc+1
                qa[ks][2 + e] = row ? __ldg(row + (16 * ks + lc + 8) / 2) : 0u;  // a4a5 / a6a7: columns + 8
            }
        }
#pragma unroll
        for (int i = 0; i < D / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
        m0 = m1 = -INFINITY;
        l0 = l1 = 0.f;
    }

    // One page: tokens [0, lim0) count for row lr and [0, lim1) for row lr+8
    // (the others are masked out of the softmax); V rows at or past vvalid
    // hold no data and are zeroed in the fragments (0 * NaN would poison).
    // Every row must have had a counted token by its first page.
    __device__ __forceinline__ void page(const uint8_t* kt, const uint8_t* vt, int lim0, int lim1, int vvalid,
                                         float qscale, int lane) {
        const int lc = (lane & 3) * 2;
        // ---- S = Q . K^T, two n8 tiles of tokens ----
        float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        {
            const int t = (lane & 7) + ((lane >> 4) << 3);
#pragma unroll
            for (int ks = 0; ks < KS; ++ks) {
                uint32_t kb[4];
                ldmatrix_x4(kb, kt + tile_off(t, 2 * ks + ((lane >> 3) & 1)));
                mma_bf16_16816(s[0], qa[ks], kb[0], kb[1]);
                mma_bf16_16816(s[1], qa[ks], kb[2], kb[3]);
            }
        }
        // s[nt][0..1]: row lr, tokens 8nt + lc, +1; s[nt][2..3]: row lr + 8
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int x = 0; x < 4; ++x) {
                const int tok = 8 * nt + lc + (x & 1);
                const int lim = x < 2 ? lim0 : lim1;
                s[nt][x] = tok < lim ? s[nt][x] * qscale : -INFINITY;
            }
        // ---- online softmax per row (the 4 lanes of a row hold its 16 tokens) ----
        float mx0 = fmaxf(fmaxf(s[0][0], s[0][1]), fmaxf(s[1][0], s[1][1]));
        float mx1 = fmaxf(fmaxf(s[0][2], s[0][3]), fmaxf(s[1][2], s[1][3]));
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
        if (__any_sync(0xffffffffu, mx0 > m0 || mx1 > m1)) {
            const float n0 = fmaxf(m0, mx0), n1 = fmaxf(m1, mx1);
            const float a0 = exp2f(m0 - n0), a1 = exp2f(m1 - n1);
            m0 = n0;
            m1 = n1;
            l0 *= a0;
            l1 *= a1;
#pragma unroll
            for (int nt = 0; nt < D / 8; ++nt) {
                o[nt][0] *= a0;
                o[nt][1] *= a0;
                o[nt][2] *= a1;
                o[nt][3] *= a1;
            }
        }
        float pr[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            pr[nt][0] = exp2f(s[nt][0] - m0);
            pr[nt][1] = exp2f(s[nt][1] - m0);
            pr[nt][2] = exp2f(s[nt][2] - m1);
            pr[nt][3] = exp2f(s[nt][3] - m1);
            l0 += pr[nt][0] + pr[nt][1];
            l1 += pr[nt][2] + pr[nt][3];
        }
        // ---- P as the A operand (k = the page's 16 tokens): bf16 high part and remainder ----
        // a0a1: (row lr, tokens lc..lc+1) = tile 0 top; a2a3: row lr+8; a4a5 / a6a7: tile 1
        uint32_t ph[4], pl[4];
#pragma unroll
        for (int x = 0; x < 4; ++x) {
            const int nt = x >> 1, half = x & 1;
            const float u = pr[nt][2 * half], v = pr[nt][2 * half + 1];
            ph[x] = float2_to_bf16x2(u, v);
            const float2 f = bf16x2_to_float2(ph[x]);
            pl[x] = float2_to_bf16x2(u - f.x, v - f.y);
        }
        // ---- O += P . V; V fragment b0b1 holds tokens lc, lc+1, b2b3 tokens lc+8, lc+9 ----
        uint32_t mlo = 0xffffffffu, mhi = 0xffffffffu;
        if (vvalid < 16) {
            mlo = (lc < vvalid ? 0x0000ffffu : 0u) | (lc + 1 < vvalid ? 0xffff0000u : 0u);
            mhi = (lc + 8 < vvalid ? 0x0000ffffu : 0u) | (lc + 9 < vvalid ? 0xffff0000u : 0u);
        }
        {
            const int t = (lane & 7) + (((lane >> 3) & 1) << 3);
#pragma unroll
            for (int nd = 0; nd < D / 16; ++nd) {
                uint32_t vb[4];
                ldmatrix_x4_trans(vb, vt + tile_off(t, 2 * nd + (lane >> 4)));
                vb[0] &= mlo;
                vb[1] &= mhi;
                vb[2] &= mlo;
                vb[3] &= mhi;
                mma_bf16_16816(o[2 * nd], ph, vb[0], vb[1]);
                mma_bf16_16816(o[2 * nd], pl, vb[0], vb[1]);
                mma_bf16_16816(o[2 * nd + 1], ph, vb[2], vb[3]);
                mma_bf16_16816(o[2 * nd + 1], pl, vb[2], vb[3]);
            }
        }
    }

    // Sums l over the 4 lanes of each row.
    __device__ __forceinline__ void finish() {
        l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
        l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
        l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
        l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    }
};

struct PrefixParams {
    CUtensorMap tmap_k;
    CUtensorMap tmap_v;
    const uint8_t* q;                   // [B][Hq][D] bf16
    const int32_t* block_tables;        // [B][M]
    const int32_t* context_lens;        // [B]
    const int32_t* group_offsets;       // [num_groups + 1]
    const int32_t* group_prefix_pages;  // [num_groups]
    int32_t num_groups, max_group_size, tiles_per_group;
    int32_t B, Hq, Hkv, NB, M;
    float qscale;                       // scale * log2(e)
    float* prefix_o;                    // [splits][B][Hq][D] partial outputs
    float2* prefix_ml;                  // [splits][B][Hq] (max logit base 2, exp-sum)
    // the step's slot-mapped append, done here (app_chunks = 0: none); the
    // decode that follows reads the new rows
    const uint4* k_new;                 // [T][Hkv][D] bf16 as 16-byte chunks
    const uint4* v_new;
    const int32_t* slot_mapping;        // [T]
    int64_t app_chunks;                 // T * Hkv * D / 8
    uint4* k_cache_w;
    uint4* v_cache_w;
};

// This CTA's slice of the step's slot-mapped append (a bit copy of 16-byte
// chunks; the rows land in the members' own blocks, never in the shared
// ones), done by the shared-prefix pass so that the decode after it sees them.
template <int D>
__device__ __forceinline__ void prefix_append_slice(const PrefixParams& p, int nthreads) {
    if (p.app_chunks <= 0) return;
    const int64_t ncta = int64_t(gridDim.x) * gridDim.y * gridDim.z;
    const int64_t lin = (int64_t(blockIdx.z) * gridDim.y + blockIdx.y) * gridDim.x + blockIdx.x;
    const int64_t per = (p.app_chunks + ncta - 1) / ncta;
    const int64_t c0 = lin * per;
    const int64_t c1 = c0 + per < p.app_chunks ? c0 + per : p.app_chunks;
    constexpr int CPR = D / 8;  // 16-byte chunks per row
    for (int64_t idx = c0 + threadIdx.x; idx < c1; idx += nthreads) {
        const int64_t t = idx / (int64_t(p.Hkv) * CPR);
        const int64_t rem = idx - t * p.Hkv * CPR;
        const int32_t slot = __ldg(p.slot_mapping + t);
        if (slot < 0) continue;
        const int64_t block = slot / 16, offset = slot - (slot / 16) * 16;
        if (block >= p.NB) {
            if (rem == 0) raise_error(PA_DEVERR_SLOT);
            continue;
        }
        const int64_t gg = rem / CPR, c = rem - gg * CPR;
        const int64_t dst = ((block * p.Hkv + gg) * 16 + offset) * CPR + c;
        p.k_cache_w[dst] = __ldg(p.k_new + idx);
        p.v_cache_w[dst] = __ldg(p.v_new + idx);
    }
}

template <int D, int NW, int RS>
struct PrefixCfg {
    static constexpr int kRow = D * 2;
    static constexpr int kTile = 16 * kRow;  // one (block, kv head) tile of 16 tokens
    static constexpr int kPanel = 16 * 128;
    static constexpr int kPage = 2 * kTile;  // K tile then V tile
    static constexpr int kRows = 16 * NW;    // query rows of a CTA
    static constexpr int kThreads = (NW + 1) * 32;
    static constexpr int kBarOff = RS * kPage;
    static constexpr int kSmemBytes = kBarOff + 2 * RS * 8 + 1024;  // + alignment slack
    static_assert(kTile % 1024 == 0, "TMA tile alignment");
    static_assert(kSmemBytes <= 232448, "shared memory per CTA");
};

// The prefix range of split z: pages [z*per, min(P, (z+1)*per)) with
// per = ceil(P / splits); the decode walks the same ranges.
__host__ __device__ __forceinline__ int prefix_split_pages(int P, int splits) { return (P + splits - 1) / splits; }

template <int D, int G, int NW, int RS>
__global__ void __launch_bounds__((NW + 1) * 32, 1) prefix_kernel(const __grid_constant__ PrefixParams p) {
    using Cfg = PrefixCfg<D, NW, RS>;
    static_assert(Cfg::kRows % G == 0, "a tile holds whole members");
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + Cfg::kBarOff);
    uint64_t* empty = full + RS;
    __shared__ int s_abort;
    volatile int* abort = &s_abort;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = blockIdx.y;

    // The decode launched after this kernel may start its set-up now; it
    // waits for this grid to complete before it reads anything written here.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    prefix_append_slice<D>(p, Cfg::kThreads);

    // ---- the group, its members and this CTA's rows and pages ----
    const int gi = int(blockIdx.x) / p.tiles_per_group;
    const int tile = int(blockIdx.x) - gi * p.tiles_per_group;
    if (gi >= p.num_groups) return;
    int first = __ldg(p.group_offsets + gi), last = __ldg(p.group_offsets + gi + 1);
    int P = __ldg(p.group_prefix_pages + gi);
    const bool report = tile == 0 && g == 0 && blockIdx.z == 0 && threadIdx.x == 0;
    if (first < 0 || last > p.B || last < first || last - first > p.max_group_size || P > p.M) {
        if (report) raise_error(PA_DEVERR_PREFIX);
        first = first < 0 ? 0 : (first > p.B ? p.B : first);
        last = last < first ? first : (last > p.B ? p.B : last);
        if (last - first > p.max_group_size) last = first + p.max_group_size;
        if (P > p.M) P = p.M;
    }
    const int nrows = (last - first) * G;
    const int row0 = tile * Cfg::kRows;
    if (P <= 0 || row0 >= nrows) return;
    const int per = prefix_split_pages(P, gridDim.z);
    const int pg0 = int(blockIdx.z) * per;
    const int pg1 = pg0 + per < P ? pg0 + per : P;
    if (pg0 >= pg1) return;
    const int npages = pg1 - pg0;
    const int leader = first;
    // warps holding at least one row of the group; the others leave now
    const int active = (nrows - row0 + 15) / 16 < NW ? (nrows - row0 + 15) / 16 : NW;

    if (threadIdx.x == 0) {
        for (int r = 0; r < RS; ++r) {
            mbar_init(&full[r], 1);
            mbar_init(&empty[r], uint32_t(active));
        }
        s_abort = 0;
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == NW) {
        // ======================= producer warp =======================
        if (lane == 0) {
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&p.tmap_k)) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&p.tmap_v)) : "memory");
        }
        const uint64_t pol = policy_evict_normal();  // every row tile of the group reads these pages
        const int32_t* bt = p.block_tables + int64_t(leader) * p.M + pg0;
        constexpr int C = RS < 32 ? RS : 32;
        bool ok = true;
        int c0 = 0;
        for (; c0 < npages; c0 += C) {
            const int n = (npages - c0) < C ? (npages - c0) : C;
            bool lane_ok = true;
            if (lane < n) {
                int32_t blk = __ldg(bt + c0 + lane);
                if (blk < 0 || blk >= p.NB) {
                    raise_error(PA_DEVERR_BLOCK_ID);
                    blk = 0;
                }
                const int i = c0 + lane, slot = i % RS;
                const uint32_t use = uint32_t(i / RS);
                if (use > 0) lane_ok = mbar_wait(&empty[slot], (use - 1) & 1, abort);
                if (lane_ok) {
                    uint8_t* st = smem + slot * Cfg::kPage;
                    mbar_arrive_expect_tx(&full[slot], Cfg::kPage);
                    tma_load_4d(st, &p.tmap_k, 0, 0, 0, blk * p.Hkv + g, &full[slot], pol);
                    tma_load_4d(st + Cfg::kTile, &p.tmap_v, 0, 0, 0, blk * p.Hkv + g, &full[slot], pol);
                }
            }
            ok = __all_sync(0xffffffffu, lane_ok);
            if (!ok) break;
        }
        if (!ok && lane == 0) {
            // Error path: let every copy this warp may have started (up to the
            // end of the failed chunk) land before shared memory is released.
            const int end = c0 + C < npages ? c0 + C : npages;
            for (int i = (end > RS ? end - RS : 0); i < end; ++i)
                mbar_wait(&full[i % RS], uint32_t(i / RS) & 1, nullptr, 20000000ull);
        }
        return;
    }
    if (warp >= active) return;

    // ========================= consumer warps =========================
    // rows wr0 .. wr0+15 of the group; row r = (member first + r / G, head g*G + r % G)
    const int wr0 = row0 + warp * 16;
    const int lr = lane >> 2, lc = (lane & 3) * 2;
    RowTile<D> rt;
    {
        const uint8_t* rows[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int r = wr0 + lr + 8 * e;
            rows[e] = r < nrows ? p.q + (int64_t(first + r / G) * p.Hq + g * G + r % G) * Cfg::kRow : nullptr;
        }
        rt.load_q(rows[0], rows[1], lane);
    }
    for (int i = 0; i < npages; ++i) {
        const int slot = i % RS;
        if (!mbar_wait(&full[slot], uint32_t(i / RS) & 1, abort)) return;
        const uint8_t* kt = smem + slot * Cfg::kPage;
        rt.page(kt, kt + Cfg::kTile, 16, 16, 16, p.qscale, lane);  // shared pages are whole
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[slot]);
    }

    // ---- the partials of the valid rows ----
    rt.finish();
    const int64_t plane = int64_t(blockIdx.z) * p.B;
#pragma unroll
    for (int e = 0; e < 2; ++e) {
        const int r = wr0 + lr + 8 * e;
        if (r >= nrows) continue;
        const int64_t idx = (plane + first + r / G) * p.Hq + g * G + r % G;
        const float l = e ? rt.l1 : rt.l0, inv = 1.f / l;
        float* dst = p.prefix_o + idx * D;
#pragma unroll
        for (int nt = 0; nt < D / 8; ++nt)
            *reinterpret_cast<float2*>(dst + nt * 8 + lc) =
                make_float2(rt.o[nt][2 * e] * inv, rt.o[nt][2 * e + 1] * inv);
        if ((lane & 3) == 0) p.prefix_ml[idx] = make_float2(e ? rt.m1 : rt.m0, l);
    }

    // ---- checks of the caller's grouping (kv head 0 only): each member holds
    // the prefix blocks in its own table and its context covers them ----
    if (g == 0) {
        const int m_lo = wr0 / G;
        const int m_hi = (wr0 + 16 < nrows ? wr0 + 16 : nrows) / G;  // members of this warp's rows
        for (int x = lane; x < (m_hi - m_lo) * npages; x += 32) {
            const int mem = first + m_lo + x / npages;
            const int j = pg0 + x % npages;
            if (__ldg(p.block_tables + int64_t(mem) * p.M + j) != __ldg(p.block_tables + int64_t(leader) * p.M + j))
                raise_error(PA_DEVERR_PREFIX);
            if (x % npages == 0 && int64_t(__ldg(p.context_lens + mem)) < int64_t(P) * 16)
                raise_error(PA_DEVERR_PREFIX);
        }
    }
}

}  // namespace pa
