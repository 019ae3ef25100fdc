"""Host bookkeeping of the Python WeightCache (no GPU): the version key it hands
the library is unique per tensor object, follows in-place updates, and a
tensor's finalizer stops tracking it when the tensor is garbage-collected.

The library keys a cached weight by its address; torch's caching allocator
reuses freed addresses for new tensors whose _version starts at 0 again, so
the key folds in a serial number that is never reused ("Cache quantized
weights for full AC", prime-rl PR #3388, Note on silent wrong numerics)."""
import gc

import torch


def test_key_version_is_per_tensor_object_and_tracks_updates():
    from mxfp8_block_scaled_cast_b200 import mx
    cache = mx.WeightCache()
    a = torch.zeros(64, 64, dtype=torch.bfloat16)
    b = a.view(64, 64)                                # another tensor object, same memory
    ka = cache.key_version(a)
    assert cache.key_version(a) == ka                 # stable while unchanged
    kb = cache.key_version(b)
    assert kb != ka and (kb >> 32) != (ka >> 32)      # a different object gets its own serial
    a.add_(1)                                         # in-place update bumps the version
    ka2 = cache.key_version(a)
    assert ka2 != ka and (ka2 >> 32) == (ka >> 32)
    assert (ka2 & 0xFFFFFFFF) == a._version
    cache.close()


def test_finalizer_stops_tracking_and_close_detaches():
    from mxfp8_block_scaled_cast_b200 import mx
    cache = mx.WeightCache()
    t = torch.ones(32, 32, dtype=torch.bfloat16)
    serial = cache.key_version(t) >> 32
    assert len(cache._tracked) == 1
    del t
    gc.collect()
    assert len(cache._tracked) == 0                   # evicted when the tensor died
    u = torch.ones(32, 32, dtype=torch.bfloat16)
    assert cache.key_version(u) >> 32 > serial        # serials are never reused
    cache.close()
    assert not cache.handle and len(cache._tracked) == 0
    del u                                             # a detached finalizer does nothing
    gc.collect()
