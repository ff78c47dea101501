"""host_streamed_paged_kvs_b200 -- host-streamed paged quantized KV attention on B200.

The product is the C-ABI library libkvs.so (include/kvs.h); ``kvs`` is its thin
ctypes binding and ``workload`` the seeded synthetic inputs.
"""
