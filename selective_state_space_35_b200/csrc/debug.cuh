// Device-side index checks of the debug build (compiled with -DSSM_DEBUG).
//
// A checked access passes its element offset through SSM_DIDX together with
// the number of elements it touches from there and the extent of the range
// it may touch, both taken from the call's shapes (a row of L tokens, a
// buffer of B*D*L elements, a checkpoint array of its documented size). When
// the access would leave that range the check counts the failure, keeps the
// first one of its translation unit (site, offset, count, extent) in a
// device-global record and returns offset 0 instead, so the access lands on
// the range's first element and the kernel runs to its end: nothing traps and
// no barrier is skipped. A check with count 0 (an access that is predicated
// off) always passes. The host reads and clears the records through
// ssm_debug_report. Without SSM_DEBUG, SSM_DIDX is its offset argument and
// neither the record nor the checks exist.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "internal.h"

// Every check site: id, printable name.
#define SSM_DEBUG_SITES(X)                                   \
  X(kDbgSelftest, "debug selftest")                          \
  X(kDbgConvRow, "conv1d row of [B][D][L]")                  \
  X(kDbgConvTok, "conv1d tokens of a row")                   \
  X(kDbgRowVec, "8-token vector access of a row")            \
  X(kDbgConvPartial, "conv1d bwd dw/dbias partials")         \
  X(kDbgConvReduce, "conv1d dw/dbias reduction")             \
  X(kDbgPackBC, "scan B/C chunk tiles")                      \
  X(kDbgS16Row, "N=16 scan row of [B][D][L]")                \
  X(kDbgS16Tok, "N=16 scan tokens of a row")                 \
  X(kDbgS16Ckpt, "N=16 scan checkpoints")                    \
  X(kDbgS16State, "N=16 scan final / summary state")         \
  X(kDbgS16BC, "N=16 scan bwd dB/dC of [B][N][L]")           \
  X(kDbgS16Part, "N=16 scan bwd dB/dC partials")             \
  X(kDbgS16Param, "N=16 scan bwd parameter partials")        \
  X(kDbgScanRow, "general scan row of [B][D][L]")            \
  X(kDbgScanCkpt, "general scan checkpoints")                \
  X(kDbgCscanRow, "complex scan row of [B][D][L]")           \
  X(kDbgCscanCkpt, "complex scan checkpoints")               \
  X(kDbgDecodeState, "decode state of [B][D][N]")            \
  X(kDbgSsdRow, "SSD token row of [B][L][H or G]")           \
  X(kDbgSsdChunkState, "SSD chunk states")                   \
  X(kDbgSsdState, "SSD final state")

namespace ssm {

#define SSM_DEBUG_ENUM(id, name) id,
enum DebugSite : int { kDbgNone = 0, SSM_DEBUG_SITES(SSM_DEBUG_ENUM) kDbgSiteCount };
#undef SSM_DEBUG_ENUM

inline const char* debug_site_name(int site) {
#define SSM_DEBUG_NAME(id, name) name,
  static const char* const names[] = {"none", SSM_DEBUG_SITES(SSM_DEBUG_NAME)};
#undef SSM_DEBUG_NAME
  return (site >= 0 && site < kDbgSiteCount) ? names[site] : "unknown";
}

#ifdef SSM_DEBUG
namespace {
__device__ DebugRecord g_debug_record;  // one per translation unit
}

__device__ __forceinline__ long long debug_index(int site, long long off, long long count,
                                                 long long extent) {
  if (count == 0 || (off >= 0 && count > 0 && off + count <= extent)) return off;
  if (atomicAdd(&g_debug_record.failures, 1ull) == 0ull) {
    g_debug_record.site = site;
    g_debug_record.offset = off;
    g_debug_record.count = count;
    g_debug_record.extent = extent;
  }
  return 0;
}

#define SSM_DIDX(site, off, count, extent)                                   \
  ::ssm::debug_index(::ssm::site, static_cast<long long>(off), static_cast<long long>(count), \
                     static_cast<long long>(extent))

// Defines debug_take_<name>: copies this translation unit's record out of the
// current device and, with reset, clears it.
#define SSM_DEBUG_TU(name)                                                        \
  cudaError_t debug_take_##name(DebugRecord* out, bool reset) {                   \
    cudaError_t e = cudaMemcpyFromSymbol(out, g_debug_record, sizeof(DebugRecord)); \
    if (e == cudaSuccess && reset) {                                              \
      const DebugRecord zero = {};                                                \
      e = cudaMemcpyToSymbol(g_debug_record, &zero, sizeof(DebugRecord));         \
    }                                                                             \
    return e;                                                                     \
  }
#else
#define SSM_DIDX(site, off, count, extent) (off)
#define SSM_DEBUG_TU(name)
#endif

}  // namespace ssm
