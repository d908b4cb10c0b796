// pa_prefill.cuh -- multi-query (chunked prefill) attention over the paged
// KV cache.
//
// Sequence b brings q_len_b query tokens, which are the last q_len_b of its
// L_b cached tokens (their K/V rows were appended before the call); query
// token i, at position pos = L_b - q_len_b + i, attends causally to tokens
// 0 .. pos.  For kv head g the rows are (token i, query head g*G + j), so a
// tile of rows against a 16-token page is a dense [rows x 16] x [16 x D]
// contraction, done on the tensor cores with the shared-prefix kernel's
// RowTile (mma.sync m16n8k16, bf16 in, fp32 accumulate).
//
// CTA = (sequence, 128-row tile, kv head).  Warp NW streams pages 0 .. the
// tile's last position of the sequence's own table (one tiled TMA copy per
// K tile and per V tile) into a ring that every consumer warp reads; warp w
// owns rows 16w .. 16w+15, masks each page per row to the tokens at or
// before the row's position, skips pages past all of its rows' positions,
// and writes its rows' bf16 output.  No key split: rows give the
// parallelism (a 512-token chunk of a 32-query-head model is 128 CTAs per
// sequence).
#pragma once

#include "pa_prefix.cuh"

namespace pa {

struct PrefillParams {
    CUtensorMap tmap_k;             // box: one (block, kv head) tile
    CUtensorMap tmap_v;
    const uint8_t* q;               // [total][Hq][D] bf16
    const int32_t* cu_q_lens;       // [B + 1]
    const int32_t* block_tables;    // [B][M]
    const int32_t* context_lens;    // [B]
    __nv_bfloat16* out;             // [total][Hq][D]
    int32_t B, Hq, Hkv, NB, M;
    int32_t tiles_per_seq;          // ceil(max_q_len * G / (16 * NW))
    float qscale;                   // scale * log2(e)
};

template <int D, int G, int NW, int RS>
__global__ void __launch_bounds__((NW + 1) * 32, 1) prefill_kernel(const __grid_constant__ PrefillParams p) {
    using Cfg = PrefixCfg<D, NW, RS>;
    static_assert(Cfg::kRows % G == 0, "a tile holds whole tokens");
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + Cfg::kBarOff);
    uint64_t* empty = full + RS;
    __shared__ int s_abort;
    volatile int* abort = &s_abort;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = blockIdx.y;

    // ---- the sequence, its query rows and the pages this tile needs ----
    const int b = int(blockIdx.x) / p.tiles_per_seq;
    const int tile = int(blockIdx.x) - b * p.tiles_per_seq;
    if (b >= p.B) return;
    const bool report = tile == 0 && g == 0 && threadIdx.x == 0;
    int32_t L = __ldg(p.context_lens + b);
    const int64_t cap = int64_t(p.M) * 16;
    if (L < 0 || L > cap) {
        if (report) raise_error(PA_DEVERR_CONTEXT);
        L = L < 0 ? 0 : int32_t(cap);
    }
    const int32_t q0 = __ldg(p.cu_q_lens + b);
    int32_t q_len = __ldg(p.cu_q_lens + b + 1) - q0;
    if (q_len < 0 || q_len > L) {  // queries must be cached tokens of the sequence
        if (report) raise_error(PA_DEVERR_CONTEXT);
        q_len = q_len < 0 ? 0 : L;
    }
    const int nrows = q_len * G;
    const int row0 = tile * Cfg::kRows;
    if (row0 >= nrows) return;
    const int first_pos = L - q_len;  // position of query token 0
    const int last_row = (row0 + Cfg::kRows < nrows ? row0 + Cfg::kRows : nrows) - 1;
    const int npages = (first_pos + last_row / G) / 16 + 1;
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
        const uint64_t pol = policy_evict_normal();  // every row tile of the sequence reads these pages
        const int32_t* bt = p.block_tables + int64_t(b) * p.M;
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
    // rows wr0 .. wr0+15; row r = (query token r / G, query head g*G + r % G)
    const int wr0 = row0 + warp * 16;
    const int lr = lane >> 2, lc = (lane & 3) * 2;
    RowTile<D> rt;
    int pos[2];
    {
        const uint8_t* rows[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int r = wr0 + lr + 8 * e;
            const bool valid = r < nrows;
            rows[e] = valid ? p.q + (int64_t(q0 + r / G) * p.Hq + g * G + r % G) * Cfg::kRow : nullptr;
            pos[e] = valid ? first_pos + r / G : first_pos;  // padding rows: any valid position
        }
        rt.load_q(rows[0], rows[1], lane);
    }
    const int warp_last = (wr0 + 15 < nrows ? wr0 + 15 : nrows - 1);
    const int warp_pages = (first_pos + warp_last / G) / 16 + 1;  // pages past these rows are skipped
    for (int i = 0; i < npages; ++i) {
        const int slot = i % RS;
        if (!mbar_wait(&full[slot], uint32_t(i / RS) & 1, abort)) return;
        if (i < warp_pages) {
            const uint8_t* kt = smem + slot * Cfg::kPage;
            const int base = 16 * i;
            const int lim0 = pos[0] - base + 1 < 16 ? pos[0] - base + 1 : 16;
            const int lim1 = pos[1] - base + 1 < 16 ? pos[1] - base + 1 : 16;
            const int vvalid = L - base < 16 ? L - base : 16;
            rt.page(kt, kt + Cfg::kTile, lim0 > 0 ? lim0 : 0, lim1 > 0 ? lim1 : 0, vvalid, p.qscale, lane);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[slot]);
    }

    // ---- bf16 output of the valid rows ----
    rt.finish();
#pragma unroll
    for (int e = 0; e < 2; ++e) {
        const int r = wr0 + lr + 8 * e;
        if (r >= nrows) continue;
        const float inv = 1.f / (e ? rt.l1 : rt.l0);
        __nv_bfloat16* dst = p.out + (int64_t(q0 + r / G) * p.Hq + g * G + r % G) * D;
#pragma unroll
        for (int nt = 0; nt < D / 8; ++nt)
            *reinterpret_cast<uint32_t*>(dst + nt * 8 + lc) =
                float2_to_bf16x2(rt.o[nt][2 * e] * inv, rt.o[nt][2 * e + 1] * inv);
    }
}

}  // namespace pa
