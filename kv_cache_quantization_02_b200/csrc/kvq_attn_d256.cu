// kvq_attn_d256.cu -- the decode attention at head dimension D = 256 (kvq_attn.cuh).
#define KVQ_ATTN_D 256
#include "kvq_attn.cuh"
