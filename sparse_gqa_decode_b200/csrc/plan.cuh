// plan.cuh -- equal-work split-KV partition of a ragged batch over CTAs.
//
// "Optimizing token dropping in sparse attention" (优化稀疏注意力中的令牌丢弃机制),
// section 5: sequences of very different lengths (128K next to 512) leave CTAs
// idle when each CTA owns a whole sequence; splitting the KV of every row
// across CTAs and reducing afterwards balances the work.  The reading used here:
//   rows = (KV head, sequence) pairs in memory order, row = kvh * B + b;
//   each row is padded to a multiple of kGranule tokens, followed by row_cost
//   more positions (a fixed work charge for its segment setup and merge; 0 for
//   a forced split and the score passes), and the rows are laid end to end
//   into one stream of W positions;
//   mode 0 cuts the stream into CTA ranges of S = max(min_chunk,
//   round_up(ceil(W / n_req), kGranule)) positions, mode 1 gives each row a CTA;
//   a segment = one CTA range intersected with the real tokens of one row;
//   segments are numbered in stream order and each yields one partial result.
// Every segment holds at least one real token; a CTA range that falls wholly
// in charged positions has no segment (the plan counts only rows whose real
// tokens meet the range).
#pragma once

#include "common.cuh"

namespace sgd {

__device__ __forceinline__ int upper_bound_i32(const int32_t *a, int n, int32_t x) {
    int lo = 0, hi = n;  // first i with a[i] > x
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (a[mid] <= x)
            lo = mid + 1;
        else
            hi = mid;
    }
    return lo;
}

// Walks the segments of one CTA in stream order.  init() is four independent loads; each
// segment then costs one 32-byte row record, which also carries what the caller needs of the
// segment's sequence, and the last segment is known without a further load.
struct SegCursor {
    const RowInfo *info;
    int R;
    int32_t end;  // CTA range end (stream position)
    int32_t pos;  // next stream position to cover
    int r;        // current row candidate
    int slot;     // slot of the next segment
    int left;     // segments still to return
    RowInfo ri;   // record of the row of the segment last returned

    __device__ void init(const PlanView &pv, int R_, int cta) {
        info = pv.row_info;
        R = R_;
        pos = pv.cta_begin[cta];
        end = pv.cta_begin[cta + 1];
        slot = pv.cta_slot0[cta];
        left = pv.cta_slot0[cta + 1] - slot;
        r = pv.cta_row0[cta];
    }

    // Next segment: row, row-local token range [t0, t1), slot.  False when done.
    __device__ bool next(int &row, int32_t &t0, int32_t &t1, int &s) {
        while (left > 0 && r < R) {
            const int4 *p = reinterpret_cast<const int4 *>(info + r);
            const int4 x = __ldg(p), y = __ldg(p + 1);
            ri.pos = x.x;
            ri.len = x.y;
            ri.seq_start = x.z;
            ri.seq_len = x.w;
            ri.len_start = y.x;
            ri.part0 = y.y;
            ri.slot0 = y.z;
            ri.nseg = y.w;
            const int32_t lo = max(pos, ri.pos), hi = min(end, ri.pos + max(ri.len, 0));
            ++r;
            if (hi > lo) {
                row = r - 1;
                t0 = lo - ri.pos;
                t1 = hi - ri.pos;
                s = slot++;
                --left;
                pos = hi;
                return true;
            }
        }
        return false;
    }
};

}  // namespace sgd
