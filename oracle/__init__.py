"""fp64 CPU oracle for the FlashNorm path. Test infrastructure only: the library never imports it."""
