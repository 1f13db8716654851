"""Float64 CPU oracle for TPLA decode: test infrastructure, never the product path."""
