"""B200-native PagedAttention decode hot path.

* ``pagedattn`` -- ctypes binding of libpagedattn.so: ``pa_reshape_and_cache``,
  ``pa_decode``, ``pa_copy_blocks`` and the host ``BlockAllocator``;
* ``runner``    -- a step driver that runs sequence events through the
  allocator and the kernels;
* ``build``     -- compiles csrc/ for sm_100a into libpagedattn.so.

Importing the package does not load the library; importing ``pagedattn``
does, and fails if it has not been built.
"""

__all__ = ["pagedattn", "runner", "build"]
