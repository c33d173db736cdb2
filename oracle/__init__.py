"""CPU oracle for the JoLT compress -> decompress path (test infrastructure only;
the CUDA library neither imports nor calls it)."""
