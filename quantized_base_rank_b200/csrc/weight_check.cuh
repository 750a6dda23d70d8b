// Host-side validity of a quantised-weight descriptor, for the forward entries that wrap
// the fused linear (the LoRDBA and Walsh-Hadamard adapters). They run a preparation
// kernel before the linear itself, so they check the weight up front with the same rules
// and statuses as the linear's own check, and a bad descriptor launches nothing:
//   N >= 1, K >= 64, codes non-null and 16-byte aligned            else QL_ERR_INVALID_ARG
//   K a multiple of 64, N a multiple of 8                           else QL_ERR_UNSUPPORTED
//   NF4+DQ: qabsmax, group_scale and mean present; int8: absmax present and 4-byte
//   aligned; any other format                                       QL_ERR_INVALID_ARG
#pragma once

#include "common.cuh"

namespace qlb {

inline ql_status weight_desc_status(const ql_weight* w) {
  if (!w || w->N < 1 || w->K < 64 || !w->codes || !aligned(w->codes, 16)) return QL_ERR_INVALID_ARG;
  if (w->K % 64 != 0 || w->N % 8 != 0) return QL_ERR_UNSUPPORTED;
  if (w->fmt == QL_FMT_NF4_DQ) return (w->qabsmax && w->group_scale && w->mean) ? QL_OK : QL_ERR_INVALID_ARG;
  if (w->fmt == QL_FMT_INT8_B64) return (w->absmax && aligned(w->absmax, 4)) ? QL_OK : QL_ERR_INVALID_ARG;
  return QL_ERR_INVALID_ARG;
}

}  // namespace qlb
