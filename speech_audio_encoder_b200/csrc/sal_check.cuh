// Bounds-checked build of the library (compiled with SAL_CHECKED into libsal_checked.so),
// a stand-in for a memory checker on machines where none may run.
//
// Before each launch the host declares the byte ranges of the buffers that launch may
// touch (ck_declare: base, length, whether it may be written). Every plain global load
// or store in a kernel passes the address it accesses through SAL_CK_LD / SAL_CK_ST. In
// the checked build an access that does not lie wholly inside one declared range, or a
// store into a read-only one, is counted in a device-side report together with the lowest
// such address and the file and line of the access, and is sent to a scratch sink
// instead, so the kernel carries on without touching memory outside its buffers. The host
// reads the report with sal_check_report. In the normal build both macros are the
// address itself and nothing else changes.
//
// Bulk tensor copies (TMA loads, stores and reduce-adds) are not routed through the
// check: the hardware clips every box to the extents of its tensor map, which the host
// builds from the same shapes it declares.
#pragma once

#include <stdint.h>

namespace sal {

constexpr int kCkSpans = 16;

struct CkReport {
  unsigned long long count;    // accesses outside the declared ranges
  unsigned long long min_key;  // lowest such address << 16 | file << 12 | line
  unsigned long long min_seq;  // the earliest launch (sequence number) that made one
};

struct CkTable {
  unsigned long long lo[kCkSpans], hi[kCkSpans];  // byte ranges [lo, hi)
  unsigned int writable;                           // bit i: range i may be stored to
  int n;
  unsigned long long seq;  // this launch's sequence number (sal_launch_count before it)
  CkReport* report;
  void* sink;  // kCkSinkBytes of scratch that redirected accesses use
};
constexpr unsigned kCkSinkBytes = 256;

#ifdef SAL_CHECKED
// sal_api.cu: record a range for the next launch on this thread; the launch takes the
// table (and clears it) in ck_take, which fails if the report cannot be set up.
void ck_declare(const void* p, uint64_t bytes, bool writable);
bool ck_take(CkTable* t);
#else
inline void ck_declare(const void*, uint64_t, bool) {}
#endif

}  // namespace sal

#ifndef SAL_CK_FILE
#define SAL_CK_FILE 0
#endif

#if defined(SAL_CHECKED) && defined(__CUDACC__)
// One table per translation unit (the library is built without relocatable device code),
// written by that unit's launches.
static __device__ sal::CkTable sal_ck_table;

namespace sal {
template <bool STORE, typename T>
__device__ __forceinline__ T* ck_access(T* p, unsigned bytes, unsigned site) {
  const unsigned long long a = reinterpret_cast<unsigned long long>(p);
  const CkTable& t = sal_ck_table;
  for (int i = 0; i < t.n; ++i)
    if (a >= t.lo[i] && a + bytes <= t.hi[i] && (!STORE || ((t.writable >> i) & 1u))) return p;
  if (t.report != nullptr) {
    atomicAdd(&t.report->count, 1ull);
    atomicMin(&t.report->min_key, (a << 16) | site);
    atomicMin(&t.report->min_seq, t.seq);
  }
  return reinterpret_cast<T*>(t.sink);
}
}  // namespace sal

#define SAL_CK_LD(p, n) (::sal::ck_access<false>((p), (n), (SAL_CK_FILE << 12) | __LINE__))
#define SAL_CK_ST(p, n) (::sal::ck_access<true>((p), (n), (SAL_CK_FILE << 12) | __LINE__))
#else
#define SAL_CK_LD(p, n) (p)
#define SAL_CK_ST(p, n) (p)
#endif
