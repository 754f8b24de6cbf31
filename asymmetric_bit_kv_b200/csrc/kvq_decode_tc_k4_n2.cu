// decode_tc_kernel instances with 4-bit keys and 2 key n-tile(s).
#define KVQ_TC_KB 4
#define KVQ_TC_NKT 2
#include "kvq_decode_tc_inst.cuh"
