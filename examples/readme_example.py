"""The usage example README.md quotes: quantize a K/V cache to 4-bit codes and back,
encode a window to E5M2, and run decode attention straight from the 4-bit cache.
Needs a B200 (sm_100a) and the built library."""
import torch

import kv_cache_quantization_fp16_b200 as kvq

B, S, H, D = 4, 4096, 8, 128
k = torch.randn(B, S, H, D, device="cuda").half(); v = torch.randn_like(k)
codes, scales = kvq.q_shapes((B, S, H, D), 4)
kc, vc = (torch.empty(codes, dtype=torch.uint8, device="cuda") for _ in range(2))
ks, vs = (torch.empty(scales, dtype=torch.float16, device="cuda") for _ in range(2))
kvq.fp16_to_q_kv(k, kc, ks, v, vc, vs, B, 0, S, wbits=4)   # quantize positions [0, S)
kvq.q_to_fp16_kv(kc, k, ks, vc, v, vs, B, 0, S, wbits=4)   # dequantize back in place
k8 = torch.empty(k.shape, dtype=torch.uint8, device="cuda")
kvq.fp16_to_fp8(k, k8, B, 1024, 2048)                       # E5M2, window [1024, 3072)
q = torch.randn(B, 32, D, device="cuda").half(); out = torch.empty_like(q)
lens = torch.full((B,), S, dtype=torch.int32, device="cuda")
kvq.decode_attention_q(q, kc, ks, vc, vs, out, B, lens, 4, D ** -0.5)
assert kvq.poll_device_error() == 0                         # device-detected paging errors
