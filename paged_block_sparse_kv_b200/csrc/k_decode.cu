// k_decode.cu -- exact softmax attention over the selected pages (GQA) + split merge.
//
// Vortex paper note, section 系统设计 1: after the indexer keeps the top-k blocks, exact
// softmax attention runs on those blocks only, gathered through the page table
// (section 系统设计 2).  Section 系统设计 3's workload planning is the split of that
// work into equal chunks sized from the SM count.
//
// Work decomposition.  Every (request, KV head) row owns k selection slots; each slot
// is a page of P tokens = P/16 tiles of 16 tokens.  The rows' tiles form one flat list
// of T = rows * k * P/16 units, cut into contiguous pieces in unit order (piece_start):
// Ws pieces of equal length over the first Us units, one per warp of a persistent grid,
// then (planned split only) smaller equal pieces over the rest, which a warp takes as
// soon as it is done with its previous piece, from a counter the step's scorer zeroed
// (or round robin over the warps when there is no counter).  Warps that drew slow pages
// then take fewer of the late pieces, so the launch ends closer to the mean warp's time.
// A piece may end inside one row and continue in the next: for every row it touches it
// writes one partial (unnormalised o, running max, running sum) to the workspace at slot
// (row + piece), an index that is unique because pieces are contiguous and ordered.  The
// merge kernel combines a row's partials in piece order with the log-sum-exp rule.  The
// result therefore depends only on the selection and the piece layout, never on where
// the pages live in the pool or which warp took which piece.
//
// Per warp: a ring of DEC_STAGES stages in shared memory, each holding one K tile and
// one V tile (16 tokens x D bf16 each), each filled by one TMA tensor load (128-byte
// swizzle; a 4-D view lands the tile as D / 64 consecutive boxes of 16 rows x 64 columns)
// that completes on a per-stage mbarrier.  A warp whose next tile has not landed sleeps in
// mbarrier try_wait rather than spinning, so the SM's other warps get the issue slots.  Unit metadata (selected
// page, physical page, valid tokens) is resolved 32 units at a time, one per lane.
// Per tile: S^T = K Q^T with mma.m16n8k16 (tokens x heads, heads padded to 8 per
// n-tile), online softmax in base 2, P^T moved into the B-operand layout with
// movmatrix, O^T += V^T P^T with ldmatrix.trans for V.  Value rows past the request's
// length are zeroed in registers, so NaN in unused slots cannot leak.
#include <type_traits>

#include "vx_attend.cuh"

namespace vx {

template <bool LATE>
struct TileMeta {
    int32_t row;
    int32_t nvalid;
    int32_t piece;  // the piece the tile belongs to (split with late pieces)
};
template <>
struct TileMeta<false> {
    int32_t row;
    int32_t nvalid;
};

__device__ __forceinline__ Resolved resolve_unit(const DecodeArgs &a, int64_t u, int64_t u_end) {
    Resolved rs{0, 0, 0, 0, false};
    if (u >= u_end) return rs;
    const int64_t r = u / a.units_per_row;
    const int64_t rem = u - r * a.units_per_row;
    const int i = static_cast<int>(rem / a.tiles_per_page);
    const int sub = static_cast<int>(rem - (int64_t)i * a.tiles_per_page);
    const int b = static_cast<int>(r / a.Hkv), h = static_cast<int>(r % a.Hkv);
    rs.row = static_cast<int32_t>(r);
    const int32_t L = a.seq_lens[b];
    if (L < 1 || L > a.max_pages * a.P) return rs;  // reported by the top-k kernel
    const int32_t j = a.sel[r * a.k + i];
    if (j < 0) return rs;
    const int n = ceil_div(L, a.P);
    if (j >= n) {
        set_err(a.err, VX_DATA_BAD_SELECTION);
        return rs;
    }
    const int tok0 = j * a.P + sub * DEC_TILE;
    const int nvalid = min(DEC_TILE, L - tok0);
    if (nvalid <= 0) return rs;
    const int32_t phys = a.page_indices[a.page_ptr[b] + j];
    if (phys < 0 || phys >= a.num_pool_pages) {
        set_err(a.err, VX_DATA_BAD_PAGE_ID);
        return rs;
    }
    rs.z = phys * a.Hkv + h;
    rs.y = sub * DEC_TILE;
    rs.nvalid = nvalid;
    rs.valid = true;
    return rs;
}

// LATE: the split has late pieces (a.chunks > a.static_chunks).  Without them a warp's static
// piece is all it does and the kernel runs the plain one-chunk-per-warp loop (the piece
// bookkeeping cost the headline and long-context steps 0.4-2 us when compiled in).
template <int D, int NT, bool LATE>
__global__ void __launch_bounds__(DEC_WARPS * 32, 1)
    k_decode_gqa(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                 const DecodeArgs a) {
    constexpr int KB = D / 64;                      // 64-column TMA boxes per tile
    constexpr int BOX_BYTES = DEC_TILE * 128;       // 16 rows x 128 bytes
    constexpr int TILE_BYTES = KB * BOX_BYTES;      // 16 x D bf16
    constexpr int STAGE_BYTES = 2 * TILE_BYTES;     // K tile + V tile
    constexpr int MT = D / 16;                      // 16-dim steps

    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;  // 128-byte swizzle wants 1 KB alignment
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g4 = lane >> 2, q4 = lane & 3;
    const uint32_t stage0 = base + (uint32_t)(warp * DEC_STAGES) * STAGE_BYTES;
    const uint32_t bar0 = base + (uint32_t)(DEC_WARPS * DEC_STAGES) * STAGE_BYTES + (uint32_t)(warp * DEC_STAGES) * 8u;
    TileMeta<LATE> *meta = reinterpret_cast<TileMeta<LATE> *>(smem_raw + (base - raw) + DEC_WARPS * DEC_STAGES * STAGE_BYTES +
                                                  DEC_WARPS * DEC_STAGES * 8) +
                     warp * DEC_STAGES;

    if (lane == 0) {
        for (int s = 0; s < DEC_STAGES; ++s) mbar_init(bar0 + 8u * s, 1);
        fence_mbar_init();
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
    }
    __syncwarp();

    const int64_t wid = (int64_t)blockIdx.x * DEC_WARPS + warp;
    if (wid >= a.static_chunks) return;
    // ---- per-row state
    uint32_t qf[NT][MT][2];
    float acc[NT][MT][4];
    float m_run[NT][2], l_run[NT][2];

    // partial of row `r` (at least one tile attended) for piece `c`: slot r + c
    auto write_partial = [&](int64_t r, int64_t c) {
        const int64_t slot = r + c;
        float lt[NT][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                float v = l_run[nt][i];
                v += __shfl_xor_sync(FULL, v, 4);
                v += __shfl_xor_sync(FULL, v, 8);
                v += __shfl_xor_sync(FULL, v, 16);
                lt[nt][i] = v;
            }
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int head = nt * 8 + 2 * q4 + (e & 1);
                    const int dim = mt * 16 + g4 + 8 * (e >> 1);
                    if (head < a.G) a.o_part[(slot * a.G + head) * a.Dv + dim] = acc[nt][mt][e];
                }
        if (g4 == 0) {
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const int head = nt * 8 + 2 * q4 + i;
                    if (head < a.G) {
                        float *ml = a.ml_part + (slot * a.G + head) * 2;
                        ml[0] = m_run[nt][i];
                        ml[1] = lt[nt][i];
                    }
                }
        }
    };
    // every row that piece c touches starts with an empty partial (max -inf, sum 0); rows
    // with attended tiles get theirs overwritten later by this same warp
    auto start_row = [&](int64_t r) {
        const int b = static_cast<int>(r / a.Hkv), h = static_cast<int>(r % a.Hkv);
        const __nv_bfloat16 *qb = a.q + ((size_t)b * a.Hq + (size_t)h * a.G) * D;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            const int head = nt * 8 + g4;
#pragma unroll
            for (int kk = 0; kk < MT; ++kk) {
                if (head < a.G) {
                    const uint32_t *qp = reinterpret_cast<const uint32_t *>(qb + (size_t)head * D + kk * 16 + 2 * q4);
                    qf[nt][kk][0] = qp[0];
                    qf[nt][kk][1] = qp[4];  // +8 dims
                } else {
                    qf[nt][kk][0] = 0u;
                    qf[nt][kk][1] = 0u;
                }
            }
#pragma unroll
            for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[nt][mt][e] = 0.f;
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                m_run[nt][i] = -INFINITY;
                l_run[nt][i] = 0.f;
            }
        }
    };

    if constexpr (!LATE) {
        // one static piece per warp: the even split
        const int64_t c = wid;
        const int64_t u_begin = chunk_start(c, a.units, a.chunks);
        const int64_t u_end = chunk_start(c + 1, a.units, a.chunks);
        const int64_t row_first = u_begin / a.units_per_row;
        const int64_t row_last = (u_end - 1) / a.units_per_row;
        int64_t cur_row = -1;
        int64_t flushed_to = row_first - 1;  // rows <= flushed_to have their partial written
        auto empty_partial = [&](int64_t r) {
            if (lane < a.G) {
                float *ml = a.ml_part + ((r + c) * a.G + lane) * 2;
                ml[0] = -INFINITY;
                ml[1] = 0.f;
            }
        };
        // The first row's query is read before waiting on the previous kernel: the query is an
        // input of the call, complete before this grid starts (the grid runs either in plain
        // stream order or after the top-k kernel, which itself starts after the scorer ends).
        // Only the selection is written by the previous kernel.
        start_row(row_first);
        cur_row = row_first;
        pdl_wait();

        // ---- pipeline
        int64_t batch = u_begin;
        Resolved rs = resolve_unit(a, batch + lane, u_end);
        uint32_t pending = __ballot_sync(FULL, rs.valid);
        uint32_t issued = 0, consumed = 0;
        bool failed = false;

        for (;;) {
            // issue loads until the ring is full or the chunk is exhausted
            while (!failed && issued - consumed < DEC_STAGES) {
                if (pending == 0) {
                    batch += 32;
                    if (batch >= u_end) break;
                    rs = resolve_unit(a, batch + lane, u_end);
                    pending = __ballot_sync(FULL, rs.valid);
                    continue;
                }
                const int src = __ffs(pending) - 1;
                pending &= pending - 1;
                const int32_t row = __shfl_sync(FULL, rs.row, src);
                const int32_t z = __shfl_sync(FULL, rs.z, src);
                const int32_t y = __shfl_sync(FULL, rs.y, src);
                const int32_t nv = __shfl_sync(FULL, rs.nvalid, src);
                const int st = static_cast<int>(issued % DEC_STAGES);
                if (lane == 0) {
                    meta[st].row = row;
                    meta[st].nvalid = nv;
                    const uint32_t bar = bar0 + 8u * st;
                    const uint32_t sK = stage0 + (uint32_t)st * STAGE_BYTES;
                    // no proxy fence: this stage's earlier shared-memory reads have completed,
                    // their values were consumed before the __syncwarp that released the stage
                    mbar_arrive_expect_tx(bar, STAGE_BYTES);
                    tma_load_4d(sK, &tmK, 0, y, 0, z, bar);
                    tma_load_4d(sK + TILE_BYTES, &tmV, 0, y, 0, z, bar);
                }
                __syncwarp();
                ++issued;
            }
            // next tile (or the end of the chunk: row = row_last + 1)
            int64_t row = row_last + 1;
            int nvalid = 0;
            int st = 0;
            if (!failed && consumed != issued) {
                st = static_cast<int>(consumed % DEC_STAGES);
                if (!__all_sync(FULL, mbar_wait_sleep(bar0 + 8u * st, (consumed / DEC_STAGES) & 1u))) {
                    // a load did not arrive in time: report, let every issued load land and
                    // finish the remaining rows as empty
                    if (lane == 0) set_err(a.err, VX_DATA_TIMEOUT);
                    for (uint32_t i = consumed; i < issued; ++i)
                        (void)mbar_wait_bounded(bar0 + 8u * (i % DEC_STAGES), (i / DEC_STAGES) & 1u);
                    failed = true;
                    cur_row = -1;
                } else {
                    row = meta[st].row;
                    nvalid = meta[st].nvalid;
                }
            }
            if (row != cur_row) {
                if (cur_row >= 0) {
                    write_partial(cur_row, c);
                    flushed_to = cur_row;
                }
                for (int64_t r = flushed_to + 1; r < row; ++r) empty_partial(r);
                flushed_to = row - 1;
                if (row > row_last) break;
                start_row(row);
                cur_row = row;
            }

            const uint32_t sK = stage0 + (uint32_t)st * STAGE_BYTES;
            attend_tile<D, NT>(sK, sK + TILE_BYTES, nvalid, a.scale_log2, qf, acc, m_run, l_run, lane);
            __syncwarp();  // every lane is done with this stage before it is refilled
            ++consumed;
        }
    } else {
        auto p_start = [&](int64_t c) -> int64_t {
            return piece_start(c, a.units, a.static_units, a.static_chunks, a.chunks);
        };
        // the next piece this warp takes after its static one (warp-uniform): from the counter,
        // or round robin over the warps
        int64_t rr_next = a.static_chunks + wid;
        auto next_piece = [&]() -> int64_t {
            if (a.piece_ctr) {
                unsigned v = 0;
                if (lane == 0) v = atomicAdd(a.piece_ctr, 1u);
                return a.static_chunks + (int64_t)__shfl_sync(FULL, v, 0);
            }
            const int64_t c = rr_next;
            rr_next += a.static_chunks;
            return c;
        };

        auto empty_piece = [&](int64_t c) {
            const int64_t u0 = p_start(c), u1 = p_start(c + 1);
            for (int64_t r = u0 / a.units_per_row; r <= (u1 - 1) / a.units_per_row; ++r)
                if (lane < a.G) {
                    float *ml = a.ml_part + ((r + c) * a.G + lane) * 2;
                    ml[0] = -INFINITY;
                    ml[1] = 0.f;
                }
            __syncwarp();
        };
        // The first row's query is read before waiting on the previous kernel: the query is an
        // input of the call, complete before this grid starts (the grid runs either in plain
        // stream order or after the top-k kernel, which itself starts after the scorer ends).
        // Only the selection is written by the previous kernel.
        // The static piece's empty partials are written before the wait as well: the workspace is
        // not touched by the previous kernel (the top-k, or nothing in plain stream order).
        int64_t fc = wid, batch = p_start(wid), f_end = p_start(wid + 1);
        int64_t cur_row = batch / a.units_per_row, cur_pc = wid;  // (row, piece) being accumulated
        start_row(cur_row);
        empty_piece(fc);
        pdl_wait();

        // ---- pipeline: the filler resolves and issues the units of piece fc in [batch, f_end),
        // then takes the next piece; the consumer attends tile after tile
        bool fill_done = false;
        Resolved rs = resolve_unit(a, batch + lane, f_end);
        uint32_t pending = __ballot_sync(FULL, rs.valid);
        uint32_t issued = 0, consumed = 0;
        bool failed = false;

        for (;;) {
            // issue loads until the ring is full or no piece is left
            while (!failed && issued - consumed < DEC_STAGES) {
                if (pending == 0) {
                    batch += 32;
                    if (batch >= f_end) {
                        if (fill_done) break;
                        const int64_t c = next_piece();
                        if (c >= a.chunks) {
                            fill_done = true;
                            break;
                        }
                        fc = c;
                        batch = p_start(c);
                        f_end = p_start(c + 1);
                        empty_piece(c);
                    }
                    rs = resolve_unit(a, batch + lane, f_end);
                    pending = __ballot_sync(FULL, rs.valid);
                    continue;
                }
                const int src = __ffs(pending) - 1;
                pending &= pending - 1;
                const int32_t row = __shfl_sync(FULL, rs.row, src);
                const int32_t z = __shfl_sync(FULL, rs.z, src);
                const int32_t y = __shfl_sync(FULL, rs.y, src);
                const int32_t nv = __shfl_sync(FULL, rs.nvalid, src);
                const int st = static_cast<int>(issued % DEC_STAGES);
                if (lane == 0) {
                    meta[st].row = row;
                    meta[st].nvalid = nv;
                    meta[st].piece = static_cast<int32_t>(fc);
                    const uint32_t bar = bar0 + 8u * st;
                    const uint32_t sK = stage0 + (uint32_t)st * STAGE_BYTES;
                    // no proxy fence: this stage's earlier shared-memory reads have completed,
                    // their values were consumed before the __syncwarp that released the stage
                    mbar_arrive_expect_tx(bar, STAGE_BYTES);
                    tma_load_4d(sK, &tmK, 0, y, 0, z, bar);
                    tma_load_4d(sK + TILE_BYTES, &tmV, 0, y, 0, z, bar);
                }
                __syncwarp();
                ++issued;
            }
            // next tile, or the end (row -1)
            int64_t row = -1, pc = -1;
            int nvalid = 0;
            int st = 0;
            if (!failed && consumed != issued) {
                st = static_cast<int>(consumed % DEC_STAGES);
                if (!__all_sync(FULL, mbar_wait_sleep(bar0 + 8u * st, (consumed / DEC_STAGES) & 1u))) {
                    // a load did not arrive in time: report, let every issued load land, drop the
                    // partial in progress (its slot keeps its empty partial) and give every piece
                    // this warp would still have taken its empty partials
                    if (lane == 0) set_err(a.err, VX_DATA_TIMEOUT);
                    for (uint32_t i = consumed; i < issued; ++i)
                        (void)mbar_wait_bounded(bar0 + 8u * (i % DEC_STAGES), (i / DEC_STAGES) & 1u);
                    failed = true;
                    cur_row = -1;
                    while (!fill_done) {
                        const int64_t c = next_piece();
                        if (c >= a.chunks) fill_done = true;
                        else empty_piece(c);
                    }
                } else {
                    row = meta[st].row;
                    nvalid = meta[st].nvalid;
                    pc = meta[st].piece;
                }
            }
            if (row != cur_row || pc != cur_pc) {
                if (cur_row >= 0) write_partial(cur_row, cur_pc);
                if (row < 0) break;
                start_row(row);
                cur_row = row;
                cur_pc = pc;
            }

            const uint32_t sK = stage0 + (uint32_t)st * STAGE_BYTES;
            attend_tile<D, NT>(sK, sK + TILE_BYTES, nvalid, a.scale_log2, qf, acc, m_run, l_run, lane);
            __syncwarp();  // every lane is done with this stage before it is refilled
            ++consumed;
        }
    }
}

// Merge: one warp per (row, query head of the group, slice of 32*PER output dims), PER
// consecutive dims per lane.  The row's partials are those of the chunks c_lo..c_hi that
// touch it (slot row + c).  Partials are taken GROUP at a time: every lane reads its dims
// of GROUP outputs, and lane i reads partial i's (max, sum), all loads issued before any
// is used, so a row with up to GROUP partials costs one round trip.  The common max comes
// first (over all partials), then the weighted outputs are summed in partial order.  The
// launcher picks PER = 1 (more warps, for few rows with many partials) or a wider slice
// (fewer warps: for many rows with few partials, or when the narrow shape would not fit in
// one wave of resident warps).
template <int DV, int PER, int GROUP>
__global__ void __launch_bounds__(256) k_merge(const DecodeArgs a) {
    pdl_wait();
    // the next grid on the stream may land now: the decode step's last kernel is short, and a
    // dependent that waits for it (such as the next step's scorer) gets its start-up done meanwhile
    pdl_trigger();
    constexpr int SLICE = 32 * PER;
    constexpr int NSLICE = DV / SLICE;
    static_assert(DV % SLICE == 0 && GROUP <= 32, "merge shape");
    using VecT = typename std::conditional<PER == 4, float4, typename std::conditional<PER == 2, float2, float>::type>::type;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t item = (int64_t)blockIdx.x * 8 + warp;
    const int64_t rows = (int64_t)a.B * a.Hkv;
    if (item >= rows * a.G * NSLICE) return;
    const int slice = static_cast<int>(item % NSLICE);
    const int64_t rg = item / NSLICE;
    const int64_t r = rg / a.G;
    const int g = static_cast<int>(rg % a.G);
    const int64_t c_lo = piece_of(r * a.units_per_row, a.units, a.static_units, a.static_chunks, a.chunks);
    const int64_t c_hi = piece_of((r + 1) * a.units_per_row - 1, a.units, a.static_units, a.static_chunks, a.chunks);
    const int np = static_cast<int>(c_hi - c_lo + 1);
    const float *ml0 = a.ml_part + ((r + c_lo) * a.G + g) * 2;                               // partial i at + i*G*2
    const float *o0 = a.o_part + ((r + c_lo) * a.G + g) * DV + slice * SLICE + lane * PER;   // partial i at + i*G*DV

    auto load_o = [&](int i) -> VecT {
        VecT z;
        memset(&z, 0, sizeof(z));
        return i < np ? *reinterpret_cast<const VecT *>(o0 + (int64_t)i * a.G * DV) : z;
    };
    // first group's outputs and (max, sum), loaded together
    VecT v[GROUP];
#pragma unroll
    for (int u = 0; u < GROUP; ++u) v[u] = load_o(u);
    const float m_first = lane < np ? ml0[(int64_t)lane * a.G * 2] : -INFINITY;
    const float l_first = lane < np ? ml0[(int64_t)lane * a.G * 2 + 1] : 0.f;

    // common max and total over all partials (lane i handles partials i, i + 32, ...)
    float M = m_first;
    for (int i = lane + 32; i < np; i += 32) M = fmaxf(M, ml0[(int64_t)i * a.G * 2]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(FULL, M, off));
    float lsum = 0.f;
    if (M != -INFINITY) {
        if (m_first != -INFINITY) lsum = exp2f(m_first - M) * l_first;
        for (int i = lane + 32; i < np; i += 32) {
            const float m = ml0[(int64_t)i * a.G * 2];
            if (m != -INFINITY) lsum += exp2f(m - M) * ml0[(int64_t)i * a.G * 2 + 1];
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) lsum += __shfl_xor_sync(FULL, lsum, off);
    // lane i keeps the weight of partial i of the first group
    const float w_first = (M == -INFINITY || m_first == -INFINITY) ? 0.f : exp2f(m_first - M);

    float o[PER];
#pragma unroll
    for (int d = 0; d < PER; ++d) o[d] = 0.f;
    // an empty partial (max -inf) holds no output values: read, then dropped
    auto add = [&](const VecT &x, float w) {
        const float *xv = reinterpret_cast<const float *>(&x);
#pragma unroll
        for (int d = 0; d < PER; ++d) o[d] += w != 0.f ? w * xv[d] : 0.f;
    };
    if (M != -INFINITY) {
#pragma unroll
        for (int u = 0; u < GROUP; ++u) add(v[u], __shfl_sync(FULL, w_first, u));
#pragma unroll 1
        for (int g0 = GROUP; g0 < np; g0 += GROUP) {  // rows with more than GROUP partials
#pragma unroll
            for (int u = 0; u < GROUP; ++u) v[u] = load_o(g0 + u);
            // lane u < GROUP computes the weight of partial g0 + u
            const int i = g0 + lane;
            const float m = (lane < GROUP && i < np) ? ml0[(int64_t)i * a.G * 2] : -INFINITY;
            const float w_lane = m == -INFINITY ? 0.f : exp2f(m - M);
#pragma unroll
            for (int u = 0; u < GROUP; ++u) add(v[u], __shfl_sync(FULL, w_lane, u));
        }
    }
    const int b = static_cast<int>(r / a.Hkv), h = static_cast<int>(r % a.Hkv);
    const size_t head = (size_t)b * a.Hq + (size_t)h * a.G + g;
    const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
    __nv_bfloat16 *dst = a.out + head * DV + slice * SLICE + lane * PER;
    if constexpr (PER == 1) {
        *dst = __float2bfloat16_rn(o[0] * inv);
    } else {
#pragma unroll
        for (int d = 0; d < PER; d += 2) *reinterpret_cast<uint32_t *>(dst + d) = pack_bf16x2(o[d] * inv, o[d + 1] * inv);
    }
    if (a.lse && lane == 0 && slice == 0)
        a.lse[head] = lsum > 0.f ? (M + log2f(lsum)) * 0.69314718055994531f : -INFINITY;
}

template <int D, int NT>
static cudaError_t launch_gqa_dn(const DecodeArgs &a, const CUtensorMap &tmK, const CUtensorMap &tmV,
                                 int grid, cudaStream_t s, bool pdl) {
    constexpr int STAGE_BYTES = 2 * DEC_TILE * D * 2;
    const bool late = a.chunks > a.static_chunks;
    const size_t smem = 1024 + (size_t)DEC_WARPS * DEC_STAGES *
                                   (STAGE_BYTES + 8 + (late ? sizeof(TileMeta<true>) : sizeof(TileMeta<false>)));
    auto kern = late ? k_decode_gqa<D, NT, true> : k_decode_gqa<D, NT, false>;
    static std::atomic<unsigned long long> done[2];
    cudaError_t e = ensure_smem_limit(kern, (int)smem, done[late ? 1 : 0]);
    if (e != cudaSuccess) return e;
    return launch_k(kern, dim3(grid), dim3(DEC_WARPS * 32), smem, s, pdl, tmK, tmV, a);
}

cudaError_t launch_decode_gqa(const DecodeArgs &a, const CUtensorMap &tmK, const CUtensorMap &tmV,
                              int grid, cudaStream_t s, bool pdl) {
    const int nt = (a.G + 7) / 8;
    if (a.Dqk == 128 && nt == 1) return launch_gqa_dn<128, 1>(a, tmK, tmV, grid, s, pdl);
    if (a.Dqk == 128 && nt == 2) return launch_gqa_dn<128, 2>(a, tmK, tmV, grid, s, pdl);
    if (a.Dqk == 64 && nt == 1) return launch_gqa_dn<64, 1>(a, tmK, tmV, grid, s, pdl);
    if (a.Dqk == 64 && nt == 2) return launch_gqa_dn<64, 2>(a, tmK, tmV, grid, s, pdl);
    return cudaErrorInvalidValue;
}

template <int DV>
static cudaError_t launch_merge_dv(const DecodeArgs &a, cudaStream_t s, bool pdl) {
    constexpr int PW = DV >= 128 ? 4 : 2;  // dims per lane of the wide shape
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const int64_t rows = (int64_t)a.B * a.Hkv;
    const int64_t wide_items = rows * a.G * (DV / (32 * PW));
    // partials of the row with the most: the pieces it spans in each region of the split
    int64_t np_max = (a.units_per_row * a.static_chunks + a.static_units - 1) / a.static_units + 1;
    if (a.chunks > a.static_chunks) {
        const int64_t ud = a.units - a.static_units, wd = a.chunks - a.static_chunks;
        np_max += (a.units_per_row * wd + ud - 1) / ud + 1;
    }
    // the narrow shapes keep 24 (16-partial groups) or 16 (32-partial groups) warps resident
    // per SM; more warps than that would run in several waves
    const int64_t narrow_items = rows * a.G * (DV / 32);
    const int64_t narrow_resident = (int64_t)sms * (np_max <= 16 ? 24 : 16);
    // the wide shape also when one 8-partial group holds every row's partials (headline: 74.3 vs
    // 74.6 us per step; long context, ~20 partials per row, is faster narrow: 67.6 vs 68.0)
    if (np_max <= 8 || wide_items >= (int64_t)sms * 8 * 4 || narrow_items > narrow_resident) {
        const dim3 grid((unsigned)((wide_items + 7) / 8));
        return launch_k(k_merge<DV, PW, 32 / PW>, grid, dim3(256), 0, s, pdl, a);
    }
    const dim3 grid((unsigned)((narrow_items + 7) / 8));
    if (np_max <= 16) return launch_k(k_merge<DV, 1, 16>, grid, dim3(256), 0, s, pdl, a);
    return launch_k(k_merge<DV, 1, 32>, grid, dim3(256), 0, s, pdl, a);
}

cudaError_t launch_merge(const DecodeArgs &a, cudaStream_t s, bool pdl) {
    switch (a.Dv) {
        case 64: return launch_merge_dv<64>(a, s, pdl);
        case 128: return launch_merge_dv<128>(a, s, pdl);
        case 512: return launch_merge_dv<512>(a, s, pdl);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace vx
