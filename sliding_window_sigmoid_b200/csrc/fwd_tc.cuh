// fwd_tc.cuh — bf16 SWAT forward on 5th-generation tensor cores (sm_100a).
//
// Computes, for one (b, h) and a 128-row query tile, the SWAT attention of
// "SWAT: Sliding Window Attention Training" (section "Balanced ALiBi", the
// attention equation): o_m = sum over the key set of act(s_mn) v_n with
// s_mn = (R_m q_m).(R_n k_n)/sqrt(d) + slope_h (m - n); act = sigmoid
// (element-wise, section "Sigmoid") or, in softmax mode, the SWA(w, s)
// softmax over the window plus sink tokens ("Sliding-window beats linear
// attention"). Only 128-key tiles that hold a key of the tile's queries are
// visited (the band, plus the sink tile): the "Sliding Window Attention"
// glossary's flash-attention entry (blocks outside the window are skipped).
//
// Persistent CTA (one per SM, it owns all 512 TMEM columns), warp roles:
//   warp 0     MMA issue (one thread): S = Q'K'^T into one of NSB TMEM buffers.
//   warp 3     MMA issue (one thread): O += P V, P read from TMEM (A operand in TMEM).
//   warp 1     TMA producer (one thread): Q tiles, K/V tiles into a ring.
//   warp 2     schedule (one thread): publishes each step ahead of time in a
//              shared-memory ring read by the MMA and TMA threads.
//   warps 4..  activation warpgroup(s) (sigmoid mode: two, or three when Q
//              and K arrive rotated and there are three S buffers, taking the
//              steps in turn; softmax mode: one): tcgen05.ld S (one query row
//              per thread, TMEM lane = row), ALiBi term, edge-tile mask (none
//              for interior tiles, whose pairs are all in the window),
//              activation, P packed to bf16 and tcgen05.st over the first 64
//              columns of its S buffer; the epilogue of each item (O: TMEM ->
//              bf16 global rows).
//   last 4     RoPE prep (when Q and K are not pre-rotated): rotate the
//              TMA-staged Q tile and each new K tile in place in shared memory
//              (SWIZZLE_128B layout), then fence.proxy.async so the tensor
//              core reads the rotated values.
// TMEM columns: S buffers [0, 128 NSB), O0 / O1 (double-buffered per item) after them.
#pragma once
#include <algorithm>
#include "common.cuh"
#include "sm100.cuh"
#include "fwd_simt.cuh"
#include "bwd_simt.cuh"
#include "rope_rows.cuh"

namespace swat {

using TcFwdArgs = FwdArgs;

template <int D>
struct FwdTcCfg {
    static constexpr int TILE_BYTES = 128 * D * 2;            // one 128-row bf16 tile
    static constexpr int HALF_BYTES = 128 * 128;              // one 64-column SW128 box
    static constexpr int NSLOT = (D == 64) ? 5 : 2;           // K/V ring slots
    static constexpr int OFF_Q = 0;                           // two Q buffers
    static constexpr int OFF_K = OFF_Q + 2 * TILE_BYTES;
    static constexpr int OFF_V = OFF_K + NSLOT * TILE_BYTES;
    static constexpr int OFF_E = OFF_V + NSLOT * TILE_BYTES;  // float2 [2][D/2]
    static constexpr int OFF_TH = OFF_E + 2 * (D / 2) * 8;    // double [D/2]
    static constexpr int OFF_BAR = OFF_TH + (D / 2) * 8;
    static constexpr int NREC = 32;                           // step records in flight (scheduler ring)
    static constexpr int RGRP = 4;                            // records published / released per barrier
    static constexpr int NBAR = 6 + 4 * NSLOT + 6 + 4 + 2 + 2 * (NREC / RGRP) + 3 + 1;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
    static constexpr int OFF_REC = OFF_MISC + 32;             // StepRec [NREC]
    static constexpr int SMEM = OFF_REC + NREC * 32 + 1024;   // + slack for 1024-B alignment
    static_assert(OFF_REC % 16 == 0 && OFF_BAR % 8 == 0, "record ring and barriers need alignment");
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr int NSB = (D == 64) ? 3 : 2;              // S buffers of 128 columns
    static constexpr uint32_t COL_O = NSB * 128;              // O0 at COL_O, O1 at COL_O + D
};

// Warp roles. Sigmoid mode runs two or three activation warpgroups that take
// the S tiles in turn (step % warpgroups), so one computes while the others
// wait for their next tiles; softmax mode keeps one, because a row's running
// maximum and sum must live in one thread.
// Warps 0 and 1 issue MMAs and TMA copies: the scheduler favours older
// (lower-numbered) warps, and these threads pace everything else. Warp 2
// walks the schedule ahead of them (StepRec ring); warp 3 issues P.V.
// Activation warpgroups start at warp 4 so that warp w owns TMEM lanes
// 32 (w % 4) .. 32 (w % 4) + 31.
template <int D, int MODE, bool PRE>
struct FwdRoles {
    // sigmoid: 2 activation warpgroups; 3 when Q and K arrive rotated (the
    // prep warps are then free) and there are 3 S buffers (d 64), so that
    // each warpgroup owns one buffer and waits on its barriers in order (an
    // mbarrier parity wait must not run a phase ahead); softmax: 1
    static constexpr int ACT_WG = (MODE == SWAT_MODE_SIGMOID_) ? ((PRE && FwdTcCfg<D>::NSB == 3) ? 3 : 2) : 1;
    static constexpr int MMA_WARP = 0;
    static constexpr int TMA_WARP = 1;
    static constexpr int SCHED_WARP = 2;
    static constexpr int PV_WARP = 3;
    static constexpr int ACT_WARP0 = 4;
    static constexpr int PREP_WARP0 = ACT_WARP0 + 4 * ACT_WG;
    static constexpr int THREADS = 32 * (PREP_WARP0 + (PRE ? 0 : 4));   // no prep warps when PRE
};
constexpr int FWD_PREP_BAR = 1;   // named barrier of the 128 prep threads

// Key tiles of a query tile: an optional sink tile (keys 0..127) when the band
// starts above it, then the band tiles from floor(max(0, i0-w+1)/128) to the
// tile holding min(N-1, i0+127).
struct TileRange {
    int n_tiles, has_sink, j0_first;
};

__device__ __forceinline__ TileRange fwd_tile_range(int i0, int N, int window, int n_sink)
{
    long long kstart = (long long)i0 - window + 1;
    if (kstart < 0) kstart = 0;
    int jf = (int)(kstart / 128) * 128;
    int jl = (min(N - 1, i0 + 127) / 128) * 128;
    int hs = (n_sink > 0 && jf > 0) ? 1 : 0;
    return {hs + (jl - jf) / 128 + 1, hs, jf};
}

__device__ __forceinline__ int fwd_tile_j0(const TileRange &r, int t)
{
    return (r.has_sink && t == 0) ? 0 : r.j0_first + (t - r.has_sink) * 128;
}

// ---------------------------------------------------------------------------
// Static schedule of a persistent CTA. Work items are (b, kv head, query
// tile, head in group), in that order (group heads fastest), so consecutive
// items share most key tiles: a query tile slides the window by one tile and
// the heads of a group read the same K/V. Each CTA takes a contiguous range
// of items. Every role walks the same sequence of steps (item, key tile):
// - RESIDENT mode (the band of a query tile fits the ring): band tile jt of a
//   sequence lives in ring slot jt mod R and is loaded (and rotated) once,
//   when the first item of the range needs it, and released after the last
//   item that needs it; the sink tile has a slot of its own.
// - STREAMING mode: every step loads its tile into the next ring slot.
// ---------------------------------------------------------------------------
struct FwdItem {
    int valid, b, kvh, h, i0, seq, lo, hi, n_tiles, has_sink;
};

struct FwdStep {
    int k, first, last, step;                // local item index, first/last tile of the item, global step
    int b, kvh, h, i0, j0;
    int slot, par, is_new, need_release, last_use;
};

struct FwdSched {
    int N, window, n_sink, Hkv, G, nQT;
    int u, u_end, u_begin;                   // item indices fit 32 bits (checked on the host)
    int nslot, r_band, resident;
    int t, k, step, stream_slot, band_slot;
    int next_load, seq_lo0, seq_slot0;       // RESIDENT mode: round-robin load pointer, slot of the sequence's first tile
    uint32_t cur_par, loaded;
    FwdItem cur, nxt;
    int p_valid, p_seq, p_lo, p_hi, p_sink;

    __device__ FwdItem item(int uu) const
    {
        FwdItem it;
        it.valid = (uu >= u_begin && uu < u_end);
        if (!it.valid) { it.seq = -1; it.lo = it.hi = it.has_sink = 0; return it; }
        const unsigned v = (unsigned)uu;
        const unsigned g = v % (unsigned)G, r = v / (unsigned)G;
        const unsigned qt = r % (unsigned)nQT, sq = r / (unsigned)nQT;
        it.seq = (int)sq;
        it.kvh = (int)(sq % (unsigned)Hkv);
        it.b = (int)(sq / (unsigned)Hkv);
        it.h = it.kvh * G + (int)g;
        it.i0 = (int)qt * 128;
        const TileRange tr = fwd_tile_range(it.i0, N, window, n_sink);
        it.lo = tr.j0_first / 128;
        it.hi = min(N - 1, it.i0 + 127) / 128;
        it.n_tiles = tr.n_tiles;
        it.has_sink = tr.has_sink;
        return it;
    }

    // Band tiles of one sequence are loaded in increasing order into
    // consecutive slots, starting at the least recently loaded slot when the
    // sequence starts in this CTA; so a load always evicts the tile loaded
    // r_band loads earlier, whose last use lies several steps back.
    __device__ void start_item()
    {
        t = 0;
        if (!resident || !cur.valid) return;
        if (!(p_valid && p_seq == cur.seq)) {
            seq_lo0 = cur.lo;
            seq_slot0 = next_load;
        }
        band_slot = (seq_slot0 + (cur.lo - seq_lo0)) % r_band;
    }

    __device__ void init(const FwdArgs &a, int nslot_, int cta, int ncta)
    {
        N = a.N; window = a.window; n_sink = a.n_sink; Hkv = a.Hkv; G = a.H / a.Hkv;
        nQT = (a.N + 127) / 128;
        const long long U = (long long)a.B * Hkv * nQT * G;
        u_begin = (int)(U * cta / ncta);
        u_end = (int)(U * (cta + 1) / ncta);
        u = u_begin;
        nslot = nslot_;
        const long long wmax = min((long long)nQT, ((long long)window + 126) / 128 + 1);
        r_band = n_sink > 0 ? nslot - 1 : nslot;
        resident = (wmax <= r_band) ? 1 : 0;
        k = 0; step = 0; stream_slot = 0; cur_par = 0; loaded = 0;
        next_load = 0; seq_lo0 = 0; seq_slot0 = 0;
        p_valid = 0; p_seq = -1; p_lo = p_hi = p_sink = 0;
        cur = item(u);
        nxt = item(u + 1);
        start_item();
    }

    __device__ __forceinline__ bool next_step(FwdStep &s)
    {
        if (u >= u_end) return false;
        s.k = k; s.step = step;
        s.first = (t == 0);
        s.last = (t == cur.n_tiles - 1);
        s.b = cur.b; s.kvh = cur.kvh; s.h = cur.h; s.i0 = cur.i0;
        const bool sink = cur.has_sink && t == 0;
        const int jt = sink ? 0 : cur.lo + t - cur.has_sink;
        s.j0 = jt * 128;
        int slot, is_new, last_use;
        if (resident) {
            const bool same_prev = p_valid && p_seq == cur.seq;
            const bool same_next = nxt.valid && nxt.seq == cur.seq;
            if (sink) {
                slot = r_band;
                is_new = !(same_prev && p_sink);
                last_use = !(same_next && nxt.has_sink);
            } else {
                slot = band_slot;
                band_slot = (band_slot + 1 == r_band) ? 0 : band_slot + 1;
                is_new = !(same_prev && p_lo <= jt && jt <= p_hi);
                last_use = !(same_next && jt >= nxt.lo);
                if (is_new) next_load = band_slot;   // the slot after the one just loaded
            }
        } else {
            slot = stream_slot;
            stream_slot = (stream_slot + 1 == nslot) ? 0 : stream_slot + 1;
            is_new = 1;
            last_use = 1;
        }
        const uint32_t bit = 1u << slot;
        if (is_new) {
            const uint32_t was = loaded & bit;
            const uint32_t par = was ? ((cur_par & bit) ^ bit) : 0u;
            cur_par = (cur_par & ~bit) | par;
            loaded |= bit;
            s.par = par ? 1 : 0;
            s.need_release = was ? 1 : 0;
        } else {
            s.par = (cur_par & bit) ? 1 : 0;
            s.need_release = 0;
        }
        s.slot = slot; s.is_new = is_new; s.last_use = last_use;
        ++step;
        if (++t == cur.n_tiles) {
            ++k; ++u;
            p_valid = cur.valid; p_seq = cur.seq; p_lo = cur.lo; p_hi = cur.hi; p_sink = cur.has_sink;
            cur = nxt;
            nxt = item(u + 1);
            start_item();
        }
        return true;
    }
};

// One step of the schedule as the single-thread roles (MMA issue, TMA) read
// it: a scheduler thread walks FwdSched ahead of them and publishes each step
// in a shared-memory ring, so their own loops carry no schedule arithmetic.
struct StepRec {
    int step, k, b, h, kvh, i0, j0;   // step < 0: end of the schedule
    uint32_t fl;                      // REC_* flags, slot << 8
};
constexpr uint32_t REC_FIRST = 1, REC_LAST = 2, REC_NEW = 4, REC_NEED_REL = 8, REC_LAST_USE = 16, REC_PAR = 32;

__device__ __forceinline__ StepRec make_rec(const FwdStep &st)
{
    StepRec r;
    r.step = st.step; r.k = st.k; r.b = st.b; r.h = st.h; r.kvh = st.kvh; r.i0 = st.i0; r.j0 = st.j0;
    r.fl = (st.first ? REC_FIRST : 0u) | (st.last ? REC_LAST : 0u) | (st.is_new ? REC_NEW : 0u) |
           (st.need_release ? REC_NEED_REL : 0u) | (st.last_use ? REC_LAST_USE : 0u) | (st.par ? REC_PAR : 0u) |
           ((uint32_t)st.slot << 8);
    return r;
}

__device__ __forceinline__ void rec_store(StepRec *ring, int rs, const StepRec &r)
{
    int4 *p = reinterpret_cast<int4 *>(ring + rs);
    p[0] = make_int4(r.step, r.k, r.b, r.h);
    p[1] = make_int4(r.kvh, r.i0, r.j0, (int)r.fl);
}

// Reads record idx. Records are published and released in groups of rgrp:
// a consumer waits once per group (an mbarrier wait costs about as much as
// an MMA, so per-record waits would starve the tensor pipe). False on abort.
__device__ __forceinline__ bool rec_read(const StepRec *ring, uint64_t *full, uint64_t *free_, int nrec, int rgrp,
                                         int idx, volatile int *abort_flag, StepRec &r)
{
    const int rs = idx % nrec, grp = rs / rgrp;
    if (rs % rgrp == 0 && !sm100::mbar_wait(full + grp, (idx / nrec) & 1, abort_flag)) return false;
    const int4 *p = reinterpret_cast<const int4 *>(ring + rs);
    const int4 x = p[0], y = p[1];
    r.step = x.x; r.k = x.y; r.b = x.z; r.h = x.w; r.kvh = y.x; r.i0 = y.y; r.j0 = y.z; r.fl = (uint32_t)y.w;
    if (rs % rgrp == rgrp - 1) sm100::mbar_arrive(free_ + grp);
    return true;
}

__device__ __forceinline__ bool named_bar_or(int id, int n, bool v)
{
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v), "r"(id), "r"(n)
        : "memory");
    return r != 0;
}

// Waits bounded by time only (used to drain in-flight async work before exit).
__device__ __forceinline__ bool mbar_wait_drain(uint64_t *bar, uint32_t parity)
{
    const uint64_t t0 = sm100::globaltimer();
    while (!sm100::mbar_try_wait(bar, parity)) {
        if (sm100::globaltimer() - t0 > SWAT_WAIT_NS) {
            record_status(-4);
            return false;
        }
    }
    return true;
}

// (cos, sin) of pos * theta with the angle reduced modulo 2*pi in fp64.
__device__ __forceinline__ float2 rope_cs(double pos_theta)
{
    const double two_pi = 6.283185307179586476925286766559;
    const double inv_two_pi = 0.15915494309189533576888376337251;
    double r = pos_theta - rint(pos_theta * inv_two_pi) * two_pi;
    float s, c;
    sincosf((float)r, &s, &c);
    return make_float2(c, s);
}

// Rotate a 128-row tile in place (SW128 layout, D/64 boxes of [128 rows][128 B]).
// Thread tau owns 16-byte chunk c = tau % (D/8) of rows r0, r0 + RS, ...
// (r0 = tau / (D/8), RS = 1024 / D), i.e. the four pairs t = 4c .. 4c+3 of
// D/8 rows. Their rotation (pos0 + r) theta_t starts from the tile base
// E0[t] = e^{i pos0 theta_t} times the thread's own e^{i r0 theta_t} and
// advances by e^{i RS theta_t} from row to row (complex products in fp32).
struct RotThread {
    float w0c[4], w0s[4], stc[4], sts[4];   // e^{i r0 theta_t}, e^{i RS theta_t}
};

template <int D>
__device__ __forceinline__ void rope_rotate_tile(uint8_t *tile, const float2 *E0, const RotThread &R, int tau)
{
    constexpr int CPR = D / 8, RS = 128 / CPR;
    const int c = tau % CPR, r0 = tau / CPR;
    float cc[4], ss[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const float2 e = E0[4 * c + q];
        cc[q] = e.x * R.w0c[q] - e.y * R.w0s[q];
        ss[q] = e.y * R.w0c[q] + e.x * R.w0s[q];
    }
    uint8_t *base = tile + (c / 8) * 16384;
    constexpr int BATCH = 8;   // rows loaded ahead of their arithmetic
#pragma unroll
    for (int kb = 0; kb < CPR; kb += BATCH) {
    uint4 v[BATCH];
#pragma unroll
    for (int k = 0; k < BATCH; ++k) {
        const int r = r0 + RS * (kb + k);
        v[k] = *reinterpret_cast<const uint4 *>(base + r * 128 + (((c % 8) ^ (r & 7)) << 4));
    }
#pragma unroll
    for (int k = 0; k < BATCH; ++k) {
        const int r = r0 + RS * (kb + k);
        uint32_t w4[4] = {v[k].x, v[k].y, v[k].z, v[k].w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float x0 = sm100::bf16lo(w4[q]), x1 = sm100::bf16hi(w4[q]);
            w4[q] = sm100::pack_bf16x2(x0 * cc[q] - x1 * ss[q], x0 * ss[q] + x1 * cc[q]);
            const float nc = cc[q] * R.stc[q] - ss[q] * R.sts[q];
            ss[q] = ss[q] * R.stc[q] + cc[q] * R.sts[q];
            cc[q] = nc;
        }
        *reinterpret_cast<uint4 *>(base + r * 128 + (((c % 8) ^ (r & 7)) << 4)) =
            make_uint4(w4[0], w4[1], w4[2], w4[3]);
    }
    }
}

// Valid key columns of one query row inside a 128-key tile: c in [lo, hi]
// (the window part: 0 <= i - j < window with hi = i - j0) or c < sh (sinks,
// which also need j <= i). Evaluated without branches.
struct RowMask {
    int lo, hi, sh;
};

__device__ __forceinline__ RowMask row_mask(int rd, int j0, int window, int n_sink)
{
    RowMask m;
    m.lo = rd - window + 1;
    m.hi = rd;
    m.sh = min(n_sink - j0, rd + 1);
    return m;
}

__device__ __forceinline__ bool col_valid(const RowMask &m, int c)
{
    return ((c >= m.lo) & (c <= m.hi)) | (c < m.sh);
}

// Validity of the 32 columns c0 .. c0+31 of one row as a bit mask (bit e =
// column c0 + e): the window part [lo, hi] and the sink part [0, sh). A few
// integer operations per 32 columns; every tile uses it, so full and edge
// tiles run the same code (no per-element index arithmetic, one code copy).
__device__ __forceinline__ uint32_t col_bits32(const RowMask &m, int c0)
{
    const int a = max(m.lo - c0, 0), z = min(m.hi - c0, 31);
    const uint32_t mw = (a <= z) ? ((0xFFFFFFFFu >> (31 - z)) & (0xFFFFFFFFu << a)) : 0u;
    const int sn = min(max(m.sh - c0, 0), 32);
    const uint32_t ms = (sn >= 32) ? 0xFFFFFFFFu : ((1u << sn) - 1u);
    return mw | ms;
}

// Sigmoid weights of 16 S columns into 8 packed bf16 pairs:
// sigma(x) = 0.5 + 0.5 tanh(x / 2), x = s/sqrt(d) + slope (i - j); with
// MASKED, columns whose bit in `m` is clear get P = 0 (without, every column
// of the chunk is in the key set).
template <bool MASKED = true>
__device__ __forceinline__ void sigmoid_chunk(const uint32_t (&v)[16], uint32_t (&pk)[8], sm100::f2 bias,
                                              sm100::f2 step2, sm100::f2 hs2, uint32_t m)
{
    const sm100::f2 half2 = {0.5f, 0.5f};
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        const sm100::f2 acc = {__uint_as_float(v[2 * e]), __uint_as_float(v[2 * e + 1])};
        const sm100::f2 x = sm100::fma2(acc, hs2, bias);
        bias = sm100::add2(bias, step2);
        const sm100::f2 th = {sm100::tanh_approx(x.x), sm100::tanh_approx(x.y)};
        sm100::f2 p = sm100::fma2(th, half2, half2);
        if (MASKED) {
            p.x = (m & (1u << (2 * e))) ? p.x : 0.f;
            p.y = (m & (1u << (2 * e + 1))) ? p.y : 0.f;
        }
        pk[e] = sm100::pack_bf16x2(p.x, p.y);
    }
}

// One 16-column chunk of P: skipped (P = 0, no arithmetic) when no key of the
// chunk is valid for any row of the warp (a warp-uniform test on the band
// edges), otherwise computed with the row's column mask.
__device__ __forceinline__ void sigmoid_chunk_any(const uint32_t (&v)[16], uint32_t s_addr, int c0,
                                                  sm100::f2 step2, sm100::f2 hs2, sm100::f2 nh2,
                                                  sm100::f2 hb2, const RowMask &mk, int rd_w0, int window,
                                                  int sink_cols)
{
    uint32_t pk[8];
    const bool all_out = ((c0 > rd_w0 + 31) || (c0 + 15 < rd_w0 - window + 1)) && (c0 >= sink_cols);
    if (all_out) {
#pragma unroll
        for (int e = 0; e < 8; ++e) pk[e] = 0u;
    } else {
        const sm100::f2 cpair = {(float)c0, (float)(c0 + 1)};
        const sm100::f2 bias = sm100::fma2(cpair, nh2, hb2);   // 0.5 slope (i - j) for columns c0, c0+1
        sigmoid_chunk(v, pk, bias, step2, hs2, col_bits32(mk, c0));
    }
    sm100::tmem_st8(s_addr + (c0 >> 1), pk);
}

// Sigmoid weights of one S tile (TMEM, one row per thread) into bf16 P over
// the first 64 columns of the same buffer; rd = i - j0 for this thread's row
// and rd_w0 for the warp's first row. The chunk loop is kept rolled (two
// chunks per iteration for the double-buffered TMEM loads) so the hot code
// stays small in the instruction cache.
__device__ __forceinline__ void act_sigmoid_tile(uint32_t s_addr, float hs, float hsl, int rd, int rd_w0, int j0,
                                                 int window, int n_sink)
{
    const RowMask mk = row_mask(rd, j0, window, n_sink);
    const sm100::f2 hs2 = {hs, hs}, step2 = {-2.f * hsl, -2.f * hsl}, nh2 = {-hsl, -hsl};
    const float hb0 = hsl * (float)rd;
    const sm100::f2 hb2 = {hb0, hb0};
    const int sink_cols = n_sink - j0;
    uint32_t v0[16], v1[16];
    sm100::tmem_ld16(s_addr, v0);
    sm100::tmem_wait_ld_dep16(v0);
#pragma unroll 1
    for (int c0 = 0; c0 < 128; c0 += 32) {
        sm100::tmem_ld16(s_addr + c0 + 16, v1);
        sigmoid_chunk_any(v0, s_addr, c0, step2, hs2, nh2, hb2, mk, rd_w0, window, sink_cols);
        sm100::tmem_wait_ld_dep16(v1);
        if (c0 + 32 < 128) sm100::tmem_ld16(s_addr + c0 + 32, v0);
        sigmoid_chunk_any(v1, s_addr, c0 + 16, step2, hs2, nh2, hb2, mk, rd_w0, window, sink_cols);
        if (c0 + 32 < 128) sm100::tmem_wait_ld_dep16(v0);
    }
}

// act_sigmoid_tile for a tile whose 128 x 128 (query, key) pairs are all in
// the key set (interior band tiles): no masks, no chunk tests.
__device__ __forceinline__ void act_sigmoid_tile_full(uint32_t s_addr, float hs, float hsl, int rd)
{
    const sm100::f2 hs2 = {hs, hs}, step2 = {-2.f * hsl, -2.f * hsl}, nh2 = {-hsl, -hsl};
    const float hb0 = hsl * (float)rd;
    const sm100::f2 hb2 = {hb0, hb0};
    uint32_t v0[16], v1[16], pk[8];
    sm100::tmem_ld16(s_addr, v0);
    sm100::tmem_wait_ld_dep16(v0);
#pragma unroll 1
    for (int c0 = 0; c0 < 128; c0 += 32) {
        sm100::tmem_ld16(s_addr + c0 + 16, v1);
        const sm100::f2 cp0 = {(float)c0, (float)(c0 + 1)};
        sigmoid_chunk<false>(v0, pk, sm100::fma2(cp0, nh2, hb2), step2, hs2, 0u);
        sm100::tmem_st8(s_addr + (c0 >> 1), pk);
        sm100::tmem_wait_ld_dep16(v1);
        if (c0 + 32 < 128) sm100::tmem_ld16(s_addr + c0 + 32, v0);
        const sm100::f2 cp1 = {(float)(c0 + 16), (float)(c0 + 17)};
        sigmoid_chunk<false>(v1, pk, sm100::fma2(cp1, nh2, hb2), step2, hs2, 0u);
        sm100::tmem_st8(s_addr + ((c0 + 16) >> 1), pk);
        if (c0 + 32 < 128) sm100::tmem_wait_ld_dep16(v0);
    }
}

// Softmax weights (log2 domain) of one S tile; returns the tile's row max
// through `mx` in pass one and writes p = 2^(x - m_used) in pass two.
// Columns outside the key set count as -inf / P = 0 (column mask).
__device__ __forceinline__ float act_softmax_max(uint32_t s_addr, float sc2, float sl2, int rd, int j0,
                                                 int window, int n_sink)
{
    float mx = -INFINITY;
    const float b2 = sl2 * (float)rd;
    const RowMask mk = row_mask(rd, j0, window, n_sink);
#pragma unroll 1
    for (int k = 0; k < 4; ++k) {
        uint32_t v[32];
        sm100::tmem_ld32(s_addr + 32 * k, v);
        const uint32_t m = col_bits32(mk, 32 * k);
        const float bk = fmaf(-sl2, (float)(32 * k), b2);
        sm100::tmem_wait_ld_dep(v);
#pragma unroll
        for (int e = 0; e < 32; ++e) {
            float x = fmaf(__uint_as_float(v[e]), sc2, fmaf(-sl2, (float)e, bk));
            x = (m & (1u << e)) ? x : -INFINITY;
            mx = fmaxf(mx, x);
        }
    }
    return mx;
}

__device__ __forceinline__ float act_softmax_p(uint32_t s_addr, float sc2, float sl2, int rd, int j0,
                                               int window, int n_sink, float m_used)
{
    float lsum = 0.f;
    const float b2 = sl2 * (float)rd;
    const RowMask mk = row_mask(rd, j0, window, n_sink);
    const bool live = m_used != -INFINITY;
#pragma unroll 1
    for (int k = 0; k < 4; ++k) {
        uint32_t v[32];
        sm100::tmem_ld32(s_addr + 32 * k, v);
        const uint32_t m = live ? col_bits32(mk, 32 * k) : 0u;
        const float bk = fmaf(-sl2, (float)(32 * k), b2);
        sm100::tmem_wait_ld_dep(v);
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            const float x0 = fmaf(__uint_as_float(v[2 * e]), sc2, fmaf(-sl2, (float)(2 * e), bk));
            const float x1 = fmaf(__uint_as_float(v[2 * e + 1]), sc2, fmaf(-sl2, (float)(2 * e + 1), bk));
            float p0 = sm100::ex2_approx(x0 - m_used), p1 = sm100::ex2_approx(x1 - m_used);
            p0 = (m & (1u << (2 * e))) ? p0 : 0.f;
            p1 = (m & (1u << (2 * e + 1))) ? p1 : 0.f;
            lsum += p0 + p1;
            pk[e] = sm100::pack_bf16x2(p0, p1);
        }
        sm100::tmem_st16(s_addr + 16 * k, pk);
    }
    return lsum;
}

// PRE: Q and K arrive RoPE-rotated (copies in a workspace): the prep
// warpgroup idles and the S MMAs wait for the TMA copies only.
template <int D, int MODE, bool PRE>
__global__ void __launch_bounds__(FwdRoles<D, MODE, PRE>::THREADS, 1)
swat_fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const FwdArgs a)
{
    using C = FwdTcCfg<D>;
    using RL = FwdRoles<D, MODE, PRE>;
    constexpr int NS = C::NSLOT;
    constexpr int FWD_PREP_WARP0 = RL::PREP_WARP0, FWD_MMA_WARP = RL::MMA_WARP, FWD_TMA_WARP = RL::TMA_WARP;
    constexpr int FWD_ACT_WARP0 = RL::ACT_WARP0;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sQ = smem + C::OFF_Q;
    uint8_t *sK = smem + C::OFF_K;
    uint8_t *sV = smem + C::OFF_V;
    float2 *sE = reinterpret_cast<float2 *>(smem + C::OFF_E);
    double *sTh = reinterpret_cast<double *>(smem + C::OFF_TH);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
    uint64_t *q_full = bars, *q_ready = bars + 2, *q_free = bars + 4;
    uint64_t *k_full = bars + 6, *k_ready = k_full + NS, *v_full = k_ready + NS, *release = v_full + NS;
    constexpr int NSB = C::NSB;
    uint64_t *s_full = release + NS, *p_full = s_full + NSB;
    uint64_t *o_full = p_full + NSB, *o_free = o_full + 2;
    uint64_t *o_upd = o_free + 2, *drain = o_upd + 1;
    constexpr int NREC = C::NREC, RGRP = C::RGRP;
    uint64_t *rec_full = drain + 1, *rec_free = rec_full + NREC / RGRP;
    uint64_t *pv_done = rec_free + NREC / RGRP, *drain_pv = pv_done + 3;
    StepRec *sRec = reinterpret_cast<StepRec *>(smem + C::OFF_REC);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

    if (threadIdx.x == 0) {
        for (int s = 0; s < 2; ++s) {
            sm100::mbar_init(q_full + s, 1);
            sm100::mbar_init(q_ready + s, 128);
            sm100::mbar_init(q_free + s, 1);
            sm100::mbar_init(o_full + s, 1);
            sm100::mbar_init(o_free + s, 128);
        }
        for (int s = 0; s < NSB; ++s) {
            sm100::mbar_init(s_full + s, 1);
            sm100::mbar_init(p_full + s, 128);
        }
        for (int s = 0; s < NS; ++s) {
            sm100::mbar_init(k_full + s, 1);
            sm100::mbar_init(k_ready + s, 128);
            sm100::mbar_init(v_full + s, 1);
            sm100::mbar_init(release + s, 1);
        }
        sm100::mbar_init(o_upd, 1);
        sm100::mbar_init(drain, 1);
        for (int s = 0; s < NREC / RGRP; ++s) {
            sm100::mbar_init(rec_full + s, 1);
            sm100::mbar_init(rec_free + s, 3);   // read by the S, P.V and TMA threads
        }
        for (int s = 0; s < NSB; ++s) sm100::mbar_init(pv_done + s, 1);
        sm100::mbar_init(drain_pv, 1);
        *abort_flag = 0;
        sm100::fence_mbar_init();
    }
    if (warp == FWD_MMA_WARP) {
        sm100::tmem_alloc(tmem_slot, C::TMEM_COLS);
        sm100::tmem_relinquish();
    }
    if (warp == FWD_TMA_WARP && lane == 0) {
        sm100::prefetch_tmap(&tm_q);
        sm100::prefetch_tmap(&tm_k);
        sm100::prefetch_tmap(&tm_v);
    }
    const int ptid = threadIdx.x - 32 * FWD_PREP_WARP0;   // 0..127 inside the prep group
    const bool is_prep = warp >= FWD_PREP_WARP0 && warp < FWD_PREP_WARP0 + 4;
    RotThread rot;
    if (!PRE && is_prep && a.use_rope) {
        if (ptid < D / 2) sTh[ptid] = exp2(-2.0 * (double)ptid / (double)D * a.log2_base);
        sm100::named_bar_sync(FWD_PREP_BAR, 128);
        constexpr int CPR = D / 8, RS = 128 / CPR;
        const int c = ptid % CPR, r0 = ptid / CPR;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const double th = sTh[4 * c + q];
            const float2 w0 = rope_cs((double)r0 * th), stp = rope_cs((double)RS * th);
            rot.w0c[q] = w0.x; rot.w0s[q] = w0.y; rot.stc[q] = stp.x; rot.sts[q] = stp.y;
        }
    }
    sm100::tc_fence_before();
    __syncthreads();
    sm100::tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    FwdSched S;
    S.init(a, NS, blockIdx.x, gridDim.x);
    FwdStep st;

    if (warp == RL::SCHED_WARP) {
        // ------------------------------------------------------------ scheduler
        if (lane == 0) {
            for (int idx = 0;; ++idx) {
                const bool more = S.next_step(st);
                const int rs = idx % NREC, grp = rs / RGRP;
                if (idx >= NREC && rs % RGRP == 0 &&
                    !sm100::mbar_wait(rec_free + grp, ((idx / NREC) - 1) & 1, abort_flag))
                    break;
                StepRec r = make_rec(st);
                if (!more) r.step = -1;
                rec_store(sRec, rs, r);
                if (rs % RGRP == RGRP - 1 || !more) sm100::mbar_arrive(rec_full + grp);
                if (!more) break;
            }
        }
    } else if (warp == FWD_TMA_WARP) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            int last_par[NS];
            for (int s = 0; s < NS; ++s) last_par[s] = -1;
            int nq = 0;
            StepRec r;
            for (int idx = 0; rec_read(sRec, rec_full, rec_free, NREC, RGRP, idx, abort_flag, r) && r.step >= 0; ++idx) {
                const int slot = (int)(r.fl >> 8), par = (r.fl & REC_PAR) ? 1 : 0;
                if (r.fl & REC_FIRST) {
                    const int qs = r.k & 1;
                    if (r.k >= 2 && !sm100::mbar_wait(q_free + qs, ((r.k - 2) >> 1) & 1, abort_flag)) break;
                    sm100::mbar_arrive_expect_tx(q_full + qs, C::TILE_BYTES);
                    for (int hh = 0; hh < D / 64; ++hh)
                        sm100::tma_load_4d(sQ + qs * C::TILE_BYTES + hh * C::HALF_BYTES, &tm_q, q_full + qs,
                                           hh * 64, r.h, r.i0, r.b);
                    // warm L2 with the next query tile of this head (a later item's Q)
                    if (r.i0 + 128 < a.N)
                        for (int hh = 0; hh < D / 64; ++hh) sm100::tma_prefetch_4d(&tm_q, hh * 64, r.h, r.i0 + 128, r.b);
                    nq = r.k + 1;
                }
                if (r.fl & REC_NEW) {
                    if ((r.fl & REC_NEED_REL) && !sm100::mbar_wait(release + slot, par ^ 1, abort_flag)) break;
                    sm100::mbar_arrive_expect_tx(k_full + slot, C::TILE_BYTES);
                    for (int hh = 0; hh < D / 64; ++hh)
                        sm100::tma_load_4d(sK + slot * C::TILE_BYTES + hh * C::HALF_BYTES, &tm_k,
                                           k_full + slot, hh * 64, r.kvh, r.j0, r.b);
                    sm100::mbar_arrive_expect_tx(v_full + slot, C::TILE_BYTES);
                    for (int hh = 0; hh < D / 64; ++hh)
                        sm100::tma_load_4d(sV + slot * C::TILE_BYTES + hh * C::HALF_BYTES, &tm_v,
                                           v_full + slot, hh * 64, r.kvh, r.j0, r.b);
                    // the next band tile usually comes next: its load then waits for a
                    // ring slot to be released, so start it towards L2 now
                    if (r.j0 + 128 < a.N)
                        for (int hh = 0; hh < D / 64; ++hh) {
                            sm100::tma_prefetch_4d(&tm_k, hh * 64, r.kvh, r.j0 + 128, r.b);
                            sm100::tma_prefetch_4d(&tm_v, hh * 64, r.kvh, r.j0 + 128, r.b);
                        }
                    last_par[slot] = par;
                }
            }
            // every issued copy must have landed before the CTA may exit
            for (int kq = max(0, nq - 2); kq < nq; ++kq) mbar_wait_drain(q_full + (kq & 1), (kq >> 1) & 1);
            for (int s = 0; s < NS; ++s)
                if (last_par[s] >= 0) {
                    mbar_wait_drain(k_full + s, last_par[s]);
                    mbar_wait_drain(v_full + s, last_par[s]);
                }
        }
    } else if (is_prep && !PRE) {
        // ------------------------------------------------------------ RoPE prep
        int ebuf = 0;
        auto make_bases = [&](int pos0) {
            ebuf ^= 1;
            if (a.use_rope && ptid < D / 2) sE[ebuf * (D / 2) + ptid] = rope_cs((double)pos0 * sTh[ptid]);
        };
        while (S.next_step(st)) {
            if (st.first) {
                const int qs = st.k & 1;
                make_bases(st.i0);
                const bool ok = sm100::mbar_wait(q_full + qs, (st.k >> 1) & 1, abort_flag);
                if (named_bar_or(FWD_PREP_BAR, 128, !ok || *abort_flag)) break;
                if (a.use_rope) rope_rotate_tile<D>(sQ + qs * C::TILE_BYTES, sE + ebuf * (D / 2), rot, ptid);
                sm100::fence_proxy_async_smem();
                sm100::mbar_arrive(q_ready + qs);
            }
            if (st.is_new) {
                make_bases(st.j0);
                const bool ok = sm100::mbar_wait(k_full + st.slot, st.par, abort_flag);
                if (named_bar_or(FWD_PREP_BAR, 128, !ok || *abort_flag)) break;
                if (a.use_rope) rope_rotate_tile<D>(sK + st.slot * C::TILE_BYTES, sE + ebuf * (D / 2), rot, ptid);
                sm100::fence_proxy_async_smem();
                sm100::mbar_arrive(k_ready + st.slot);
            }
        }
    } else if (warp == FWD_MMA_WARP || warp == RL::PV_WARP) {
        // ------------------------------------------------------------ MMA issue
        // Two issuing threads feed the tensor pipe: warp 0 issues S = Q'K'^T,
        // warp 3 issues O += P V. While one waits on an mbarrier the other's
        // MMAs keep the pipe busy. S of step s reuses the TMEM buffer of step
        // s - NSB, so it waits until that step's P.V has completed (pv_done).
        constexpr uint32_t TILE16 = C::TILE_BYTES >> 4, HALF16 = C::HALF_BYTES >> 4;
        auto mk = [](uint32_t hi, uint32_t lo) { return ((uint64_t)hi << 32) | lo; };
        if (warp == FWD_MMA_WARP && lane == 0) {
            constexpr uint32_t IDESC_S = sm100::idesc_bf16_f32(128, 128, 0, 0);
            const uint64_t dq0 = sm100::sdesc_sw128(sm100::smem_u32(sQ), 16, 1024);
            const uint64_t dk0 = sm100::sdesc_sw128(sm100::smem_u32(sK), 16, 1024);
            const uint32_t hi_k = (uint32_t)(dk0 >> 32), lo_q = (uint32_t)dq0, lo_k = (uint32_t)dk0;
            StepRec r;
            for (int idx = 0;; ++idx) {
                if (!rec_read(sRec, rec_full, rec_free, NREC, RGRP, idx, abort_flag, r) || r.step < 0) break;
                const int qs = r.k & 1, sb = r.step % NSB, slot = (int)(r.fl >> 8);
                if ((r.fl & REC_FIRST) && !sm100::mbar_wait((PRE ? q_full : q_ready) + qs, (r.k >> 1) & 1, abort_flag))
                    break;
                if ((r.fl & REC_NEW) &&
                    !sm100::mbar_wait((PRE ? k_full : k_ready) + slot, (r.fl & REC_PAR) ? 1 : 0, abort_flag))
                    break;
                if (r.step >= NSB && !sm100::mbar_wait(pv_done + sb, ((r.step / NSB) - 1) & 1, abort_flag)) break;
                sm100::tc_fence_after();
                const uint32_t lq = lo_q + (uint32_t)qs * TILE16, lk = lo_k + (uint32_t)slot * TILE16;
                const uint32_t d_s = tmem + sb * 128;
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    const uint32_t off = (ks / 4) * HALF16 + (ks % 4) * 2;
                    sm100::umma_ss(d_s, mk(hi_k, lq + off), mk(hi_k, lk + off), IDESC_S, ks > 0 ? 1u : 0u);
                }
                sm100::umma_commit(s_full + sb);
                if (r.fl & REC_LAST) sm100::umma_commit(q_free + qs);
            }
            sm100::umma_commit(drain);
            mbar_wait_drain(drain, 0);   // nothing of ours is in flight past this point
        } else if (warp == RL::PV_WARP && lane == 0) {
            constexpr uint32_t IDESC_PV = sm100::idesc_bf16_f32(128, D, 0, 1);
            const uint64_t dv0 = sm100::sdesc_sw128(sm100::smem_u32(sV), C::HALF_BYTES, 1024);
            const uint32_t hi_v = (uint32_t)(dv0 >> 32), lo_v = (uint32_t)dv0;
            StepRec p;
            for (int idx = 0;; ++idx) {
                if (!rec_read(sRec, rec_full, rec_free, NREC, RGRP, idx, abort_flag, p) || p.step < 0) break;
                const int sb = p.step % NSB, ob = p.k & 1, slot = (int)(p.fl >> 8);
                const bool first = (p.fl & REC_FIRST) != 0;
                if (!sm100::mbar_wait(p_full + sb, (p.step / NSB) & 1, abort_flag)) break;
                if ((p.fl & REC_NEW) && !sm100::mbar_wait(v_full + slot, (p.fl & REC_PAR) ? 1 : 0, abort_flag)) break;
                if (first && p.k >= 2 && !sm100::mbar_wait(o_free + ob, ((p.k - 2) >> 1) & 1, abort_flag)) break;
                sm100::tc_fence_after();
                const uint32_t lv = lo_v + (uint32_t)slot * TILE16;
                const uint32_t d_o = tmem + C::COL_O + ob * D, a_p = tmem + sb * 128;
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    sm100::umma_ts(d_o, a_p + ks * 8, mk(hi_v, lv + ks * (2048 >> 4)), IDESC_PV,
                                   (!first || ks > 0) ? 1u : 0u);
                sm100::umma_commit(pv_done + sb);
                // the K tile of this step was read by S(step), complete before P(step) existed
                if (p.fl & REC_LAST_USE) sm100::umma_commit(release + slot);
                if (MODE == SWAT_MODE_SOFTMAX_) sm100::umma_commit(o_upd);
                if (p.fl & REC_LAST) sm100::umma_commit(o_full + ob);
            }
            sm100::umma_commit(drain_pv);
            mbar_wait_drain(drain_pv, 0);
        }
        __syncwarp();
    } else if (warp >= FWD_ACT_WARP0 && warp < FWD_PREP_WARP0) {
        // ------------------------------------------------------------ activation + epilogue
        // The epilogue of an item (O: TMEM -> bf16 global rows) is deferred to
        // after this warpgroup's next tile: by then the item's last P.V has
        // long completed, so the wait for O costs nothing.
        const int aw = (warp - FWD_ACT_WARP0) / 4;       // activation warpgroup
        const uint32_t lane_base = (uint32_t)(32 * (warp % 4)) << 16;
        const int r = 32 * (warp % 4) + lane;            // query row inside the tile (= TMEM lane)
        float m_used = -INFINITY, l_sum = 0.f;           // softmax state (log2 domain)
        const float LOG2E = 1.4426950408889634f;
        struct PendO { int k, b, h, i0; };
        PendO pend{};
        bool has_pend = false;
        float pend_inv = 1.f;
        auto epilogue = [&](const PendO &p, float inv) -> bool {
            const int ob = p.k & 1;
            const bool ok = sm100::mbar_wait(o_full + ob, (p.k >> 1) & 1, abort_flag);
            if (__any_sync(0xffffffffu, !ok)) return false;
            sm100::tc_fence_after();
            const int i = p.i0 + r;
            __nv_bfloat16 *orow = reinterpret_cast<__nv_bfloat16 *>(a.o) + (((size_t)p.b * a.N + i) * a.H + p.h) * D;
            const uint32_t o_addr = tmem + lane_base + C::COL_O + ob * D;
#pragma unroll
            for (int kk = 0; kk < D / 32; ++kk) {
                uint32_t v[32];
                sm100::tmem_ld32(o_addr + 32 * kk, v);
                sm100::tmem_wait_ld_dep(v);
                if (i < a.N) {
                    uint32_t pk[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        pk[e] = sm100::pack_bf16x2(__uint_as_float(v[2 * e]) * inv, __uint_as_float(v[2 * e + 1]) * inv);
                    uint4 *dst = reinterpret_cast<uint4 *>(orow + 32 * kk);
#pragma unroll
                    for (int e = 0; e < 4; ++e) dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
                }
            }
            sm100::tc_fence_before();
            sm100::mbar_arrive(o_free + ob);
            return true;
        };
        bool good = true;
        while (good && S.next_step(st)) {
            const int sb = st.step % NSB;
            if (RL::ACT_WG > 1 && st.step % RL::ACT_WG != aw) continue;   // another warpgroup's tile
            const int i = st.i0 + r;
            const float slope = a.slopes ? __ldg(a.slopes + st.h) : 0.f;
            if (st.first) { m_used = -INFINITY; l_sum = 0.f; }
            bool ok = sm100::mbar_wait(s_full + sb, (st.step / NSB) & 1, abort_flag);
            if (__any_sync(0xffffffffu, !ok)) break;
            sm100::tc_fence_after();
            const int j0 = st.j0;
            const int rd = i - j0;
            const uint32_t s_addr = tmem + lane_base + sb * 128;
            if (MODE == SWAT_MODE_SIGMOID_) {
                const float hs = 0.5f * a.scale, hsl = 0.5f * slope;
                const int rd_w0 = st.i0 + 32 * (warp % 4) - j0;   // first row of this warp
                // every pair of the tile in the window: j0 + 127 <= i0 and i0 + 127 - j0 < w
                if (j0 + 127 <= st.i0 && st.i0 + 127 - j0 < a.window)
                    act_sigmoid_tile_full(s_addr, hs, hsl, rd);
                else
                    act_sigmoid_tile(s_addr, hs, hsl, rd, rd_w0, j0, a.window, a.n_sink);
            } else {
                const float sc2 = a.scale * LOG2E, sl2 = slope * LOG2E;
                const float mx = act_softmax_max(s_addr, sc2, sl2, rd, j0, a.window, a.n_sink);
                // keep a stale maximum while the new one exceeds it by at most 8
                // (weights stay <= 2^8); otherwise rescale this row of O and l
                const bool need = mx > m_used + 8.0f;
                const bool need_o = need && m_used != -INFINITY;
                if (__any_sync(0xffffffffu, need_o)) {
                    ok = sm100::mbar_wait(o_upd, (st.step - 1) & 1, abort_flag);
                    if (__any_sync(0xffffffffu, !ok)) break;
                    sm100::tc_fence_after();
                    const float f = need_o ? sm100::ex2_approx(m_used - mx) : 1.f;
                    const uint32_t o_addr = tmem + lane_base + C::COL_O + (st.k & 1) * D;
#pragma unroll
                    for (int kk = 0; kk < D / 32; ++kk) {
                        uint32_t v[32];
                        sm100::tmem_ld32(o_addr + 32 * kk, v);
                        sm100::tmem_wait_ld_dep(v);
#pragma unroll
                        for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * f);
                        sm100::tmem_st32(o_addr + 32 * kk, v);
                    }
                    if (need_o) l_sum *= f;
                }
                if (need) m_used = mx;
                l_sum += act_softmax_p(s_addr, sc2, sl2, rd, j0, a.window, a.n_sink, m_used);
            }
            sm100::tmem_wait_st();
            sm100::tc_fence_before();
            sm100::mbar_arrive(p_full + sb);
            if (has_pend) {
                has_pend = false;
                if (!epilogue(pend, pend_inv)) { good = false; break; }
            }
            if (st.last) {
                pend = PendO{st.k, st.b, st.h, st.i0};
                has_pend = true;
                pend_inv = (MODE == SWAT_MODE_SOFTMAX_) ? 1.f / l_sum : 1.f;
                if (MODE == SWAT_MODE_SOFTMAX_ && i < a.N)
                    a.lse[((size_t)st.b * a.H + st.h) * a.N + i] = (m_used + log2f(l_sum)) * 0.6931471805599453f;
            }
        }
        if (good && has_pend) epilogue(pend, pend_inv);
    }

    sm100::tc_fence_before();
    __syncthreads();
    sm100::tc_fence_after();
    if (warp == FWD_MMA_WARP) sm100::tmem_dealloc(tmem, C::TMEM_COLS);
}

// ---------------------------------------------------------------------------
// Host side: tensor maps and launch
// ---------------------------------------------------------------------------
typedef CUresult (*PFN_tmapEncodeTiled)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                         const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                         const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                         CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline PFN_tmapEncodeTiled tmap_encoder()
{
    static PFN_tmapEncodeTiled fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_tmapEncodeTiled>(p);
    }
    return fn;
}

// bf16 tensor [B, N, Hx, D] (BSHD) as a 4-D map (D, Hx, N, B); box = 64 x 1 x 128 x 1, SW128.
inline bool make_tmap_bshd(CUtensorMap *m, const void *ptr, int B, int N, int Hx, int D)
{
    PFN_tmapEncodeTiled enc = tmap_encoder();
    if (!enc) return false;
    cuuint64_t dims[4] = {(cuuint64_t)D, (cuuint64_t)Hx, (cuuint64_t)N, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)D * 2, (cuuint64_t)Hx * D * 2, (cuuint64_t)N * Hx * D * 2};
    cuuint32_t box[4] = {64, 1, 128, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(ptr), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

inline int num_sms()
{
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
    return n;
}

template <int D, int MODE>
inline int launch_fwd_tc_t(const FwdArgs &a, void *ws, cudaStream_t stream)
{
    using C = FwdTcCfg<D>;
    int n = 0;
    const void *qr = a.q, *kr = a.k;
    const bool pre = ws != nullptr && a.use_rope;
    if (pre) n += launch_rope_copies<D>(a.q, a.k, ws, a.B, a.H, a.Hkv, a.N, a.log2_base, stream, &qr, &kr);
    CUtensorMap tq, tk, tv;
    if (!make_tmap_bshd(&tq, qr, a.B, a.N, a.H, D) || !make_tmap_bshd(&tk, kr, a.B, a.N, a.Hkv, D) ||
        !make_tmap_bshd(&tv, a.v, a.B, a.N, a.Hkv, D))
        return -1;
    auto kern = pre ? swat_fwd_tc_kernel<D, MODE, true> : swat_fwd_tc_kernel<D, MODE, false>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) != cudaSuccess) return -1;
    const long long items = (long long)a.B * a.H * ((a.N + 127) / 128);
    if (items >= (1LL << 31)) return -1;   // the schedule decodes item indices in 32 bits
    const int grid = (int)std::min<long long>(items, (long long)num_sms());
    const int threads = pre ? FwdRoles<D, MODE, true>::THREADS : FwdRoles<D, MODE, false>::THREADS;
    kern<<<grid, threads, C::SMEM, stream>>>(tq, tk, tv, a);
    return n + 1;
}

// ws: NULL (rotate Q and K tiles in shared memory) or rope_copies_bytes()
// of device memory for rotated copies. Returns the number of kernels
// launched, or -1 on a launch-configuration error.
inline int launch_fwd_tc(const TcFwdArgs &a, void *ws, cudaStream_t stream)
{
    if (a.d == 64)
        return a.mode == SWAT_MODE_SIGMOID_ ? launch_fwd_tc_t<64, SWAT_MODE_SIGMOID_>(a, ws, stream)
                                            : launch_fwd_tc_t<64, SWAT_MODE_SOFTMAX_>(a, ws, stream);
    if (a.d == 128)
        return a.mode == SWAT_MODE_SIGMOID_ ? launch_fwd_tc_t<128, SWAT_MODE_SIGMOID_>(a, ws, stream)
                                            : launch_fwd_tc_t<128, SWAT_MODE_SOFTMAX_>(a, ws, stream);
    return -1;
}

}  // namespace swat
