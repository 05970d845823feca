// Pipeline timeline trace.  Compiled in only with -DX1CB_TRACE (the default
// build has no trace code at all): each role of the first kTraceCtas CTAs
// records the SM clock (clock64) at numbered events -- event ev of the n-th
// tile, stage or box it handles -- into a device table that the host reads
// with x1cb_trace_copy.  All events of one CTA share one SM clock, so the
// differences between them are the pipeline's waits and latencies.
#pragma once
#include <cstdint>

namespace x1cb {

constexpr int kTraceCtas = 4;
constexpr int kTraceEvents = 16;
constexpr int kTraceSeq = 1024;
constexpr int kTraceWords = kTraceCtas * kTraceEvents * kTraceSeq;

#ifdef X1CB_TRACE
__device__ __forceinline__ void trace_at(unsigned long long *table, int ev, long long n)
{
    if (table && blockIdx.x < kTraceCtas && n >= 0 && n < kTraceSeq && ev >= 0 &&
        ev < kTraceEvents)
        table[(static_cast<long long>(blockIdx.x) * kTraceEvents + ev) * kTraceSeq + n] =
            clock64();
}
#define X1CB_TRACE_AT(table, ev, n) ::x1cb::trace_at((table), (ev), (n))
#else
#define X1CB_TRACE_AT(table, ev, n) ((void)0)
#endif

}  // namespace x1cb
