// decode_tc_kernel instances with 2-bit keys and 1 key n-tile(s).
#define KVQ_TC_KB 2
#define KVQ_TC_NKT 1
#include "kvq_decode_tc_inst.cuh"
